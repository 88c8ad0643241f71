// The rest of a Mamba2 block around the bidirectional scan (optional part of the MATE block's MA branch;
// the pages name the branch's core a bidirectional Mamba2 block without listing its internals):
//   * conv_silu_kernel     causal depthwise convolution (width 4, bias) + SiLU over the x | B | C channels,
//                          along each sample's scan sequence [review rows; video rows in scan order];
//   * gate_rmsnorm_kernel  y <- (y * silu(z)) / sqrt(mean((y * silu(z))^2) + eps) * norm_w, per row, in place.
// Both are HBM-bound streams of whole rows: coalesced 16-byte vectors where the row strides allow, fp32
// arithmetic, the storage type's rounding on the way out.
#pragma once
#include "common.cuh"
#include "simt.cuh"

namespace mate {

constexpr int kConvK = 4;          // taps of the causal convolution; tap kConvK - 1 is the current row
constexpr int kConvRun = 16;       // sequence positions per thread (the window slides in registers)
constexpr float kNormEps = 1e-5f;  // epsilon of the gated RMSNorm

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T_> __device__ __forceinline__ T_ from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// V consecutive elements as fp32; one 16-byte access when V elements fill 16 bytes (the caller has
// checked the alignment), else element by element.
template <typename T_, int V>
__device__ __forceinline__ void load_vec(const T_* p, float (&f)[V]) {
  if constexpr (sizeof(T_) * V == 16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const T_* e = reinterpret_cast<const T_*>(&u);
#pragma unroll
    for (int i = 0; i < V; ++i) f[i] = to_f32(e[i]);
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i) f[i] = to_f32(p[i]);
  }
}

template <typename T_, int V>
__device__ __forceinline__ void store_vec(T_* p, const float (&f)[V]) {
  if constexpr (sizeof(T_) * V == 16) {
    uint4 u;
    T_* e = reinterpret_cast<T_*>(&u);
#pragma unroll
    for (int i = 0; i < V; ++i) e[i] = from_f32<T_>(f[i]);
    *reinterpret_cast<uint4*>(p) = u;
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i) p[i] = from_f32<T_>(f[i]);
  }
}

// SiLU with the fast divide (a few ulp; for v < -88 the quotient is 0, the value rounded to zero anyway).
__device__ __forceinline__ float silu_f(float v) { return __fdividef(v, 1.f + __expf(-v)); }

// Causal depthwise convolution + SiLU.  Sequence position i of sample b reads the source row of s (prefix
// row rrow(b, i) of s.xr for i < R, else video row vrow(b, i - R) of s.xv, row strides s.ldxr / s.ldxv)
// and writes the same row of the outputs (out_r / out_v, row stride ldo).  Channels [0, C), C a
// multiple of V.  Thread g owns channel vector g % nvec and the kConvRun positions of run g / nvec; the
// kConvK - 1 rows before its run are read again as its window's start (zero before position 0).
// w: [C][kConvK] fp32, tap kConvK - 1 on the current row; bias: [C].
template <typename T_, int V>
__global__ void __launch_bounds__(256) conv_silu_kernel(SeqRows s, int C, const float* __restrict__ w,
                                                        const float* __restrict__ bias, T_* __restrict__ out_v,
                                                        T_* __restrict__ out_r, int ldo, int nruns, int B) {
  const int nvec = C / V;
  const long long total = (long long)B * nruns * nvec;
  const int L = s.R + s.n;
  for (long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x; g < total;
       g += (long long)gridDim.x * blockDim.x) {
    const int vi = static_cast<int>(g % nvec);
    const long long rb = g / nvec;
    const int b = static_cast<int>(rb / nruns);
    const int i0 = static_cast<int>(rb - (long long)b * nruns) * kConvRun;
    const int c0 = vi * V;
    float wt[V][kConvK], bs[V];
#pragma unroll
    for (int e = 0; e < V; ++e) {
      const float4 t = __ldg(reinterpret_cast<const float4*>(w + (size_t)(c0 + e) * kConvK));
      wt[e][0] = t.x; wt[e][1] = t.y; wt[e][2] = t.z; wt[e][3] = t.w;
      bs[e] = __ldg(bias + c0 + e);
    }
    // window[k] holds position i - (kConvK - 1) + k
    float win[kConvK][V];
#pragma unroll
    for (int k = 0; k < kConvK - 1; ++k) {
      const int i = i0 - (kConvK - 1) + k;
      if (i < 0) {
#pragma unroll
        for (int e = 0; e < V; ++e) win[k][e] = 0.f;
      } else {
        const T_* src = i < s.R ? static_cast<const T_*>(s.xr) + s.rrow(b, i) * s.ldxr
                                : static_cast<const T_*>(s.xv) + s.vrow(b, i - s.R) * s.ldxv;
        load_vec<T_, V>(src + c0, win[k]);
      }
    }
    const int i_end = min(L, i0 + kConvRun);
    for (int i = i0; i < i_end; ++i) {
      const bool pre = i < s.R;
      const long long row = pre ? s.rrow(b, i) : s.vrow(b, i - s.R);
      const T_* src = pre ? static_cast<const T_*>(s.xr) + row * s.ldxr : static_cast<const T_*>(s.xv) + row * s.ldxv;
      load_vec<T_, V>(src + c0, win[kConvK - 1]);
      float o[V];
#pragma unroll
      for (int e = 0; e < V; ++e) {
        float acc = bs[e];
#pragma unroll
        for (int k = 0; k < kConvK; ++k) acc = fmaf(wt[e][k], win[k][e], acc);
        o[e] = silu_f(acc);
      }
      store_vec<T_, V>((pre ? out_r : out_v) + row * ldo + c0, o);
#pragma unroll
      for (int k = 0; k < kConvK - 1; ++k)
#pragma unroll
        for (int e = 0; e < V; ++e) win[k][e] = win[k + 1][e];
    }
  }
}

// Causal depthwise convolution + SiLU as a tiled stencil: a CTA takes kCvTP consecutive sequence positions
// x kCvTC channels of one sample, loads those rows plus the kConvK - 1 rows before them into shared memory
// (every load of the tile in flight at once, rows gathered through the scan-order map), then computes the
// outputs from shared memory.  Same result as conv_silu_kernel; needs 16-byte vectors (C % V == 0, aligned
// rows).  Dynamic shared memory: (kCvTP + kConvK - 1) * kCvTC * sizeof(T_).
constexpr int kCvTP = 64, kCvTC = 256;

template <typename T_>
__global__ void __launch_bounds__(256) conv_silu_tiled_kernel(SeqRows s, int C, const float* __restrict__ w,
                                                              const float* __restrict__ bias, T_* __restrict__ out_v,
                                                              T_* __restrict__ out_r, int ldo, int ntp, int ntc) {
  extern __shared__ __align__(16) uint8_t cv_smem[];
  T_* tile = reinterpret_cast<T_*>(cv_smem);   // [kCvTP + kConvK - 1][kCvTC]
  constexpr int V = 16 / sizeof(T_);
  constexpr int NV = kCvTC / V;                // vectors per tile row
  constexpr int RW = kCvTP + kConvK - 1;
  constexpr int NIT = (RW * NV + 255) / 256;   // tile vectors per thread
  __shared__ long long s_row[RW];              // source row of each tile row (-1 outside the sequence)
  __shared__ int s_pre[RW];                    // 1: a review-prefix row
  const int L = s.R + s.n;
  const int t = blockIdx.x;
  const int ct = t % ntc, pt = (t / ntc) % ntp, b = t / (ntc * ntp);
  const int pos0 = pt * kCvTP, ch0 = ct * kCvTC;
  for (int r = threadIdx.x; r < RW; r += blockDim.x) {
    const int i = pos0 - (kConvK - 1) + r;
    long long row = -1;
    int pre = 0;
    if (i >= 0 && i < L) {
      pre = i < s.R;
      row = pre ? s.rrow(b, i) : s.vrow(b, i - s.R);
    }
    s_row[r] = row;
    s_pre[r] = pre;
  }
  __syncthreads();
  uint4 v[NIT];
#pragma unroll
  for (int k = 0; k < NIT; ++k) {
    const int it = threadIdx.x + k * 256;
    const int r = it / NV, cv = it % NV, ch = ch0 + cv * V;
    v[k] = make_uint4(0, 0, 0, 0);
    if (it < RW * NV && ch < C) {
      const long long row = s_row[r];
      if (row >= 0) {
        const T_* src = s_pre[r] ? static_cast<const T_*>(s.xr) + row * s.ldxr : static_cast<const T_*>(s.xv) + row * s.ldxv;
        v[k] = __ldg(reinterpret_cast<const uint4*>(src + ch));
      }
    }
  }
#pragma unroll
  for (int k = 0; k < NIT; ++k) {
    const int it = threadIdx.x + k * 256;
    if (it < RW * NV) *reinterpret_cast<uint4*>(tile + (it / NV) * kCvTC + (it % NV) * V) = v[k];
  }
  __syncthreads();
  const int cv = threadIdx.x % NV, ch = ch0 + cv * V;
  if (ch >= C) return;
  float wt[V][kConvK], bs[V];
#pragma unroll
  for (int e = 0; e < V; ++e) {
    const float4 q = __ldg(reinterpret_cast<const float4*>(w + (size_t)(ch + e) * kConvK));
    wt[e][0] = q.x; wt[e][1] = q.y; wt[e][2] = q.z; wt[e][3] = q.w;
    bs[e] = __ldg(bias + ch + e);
  }
  for (int p = threadIdx.x / NV; p < kCvTP; p += blockDim.x / NV) {
    const int i = pos0 + p;
    if (i >= L) break;
    float o[V];
#pragma unroll
    for (int e = 0; e < V; ++e) o[e] = bs[e];
#pragma unroll
    for (int k = 0; k < kConvK; ++k) {   // tile row p + k holds position i - (kConvK - 1) + k
      float f[V];
      const uint4 u = *reinterpret_cast<const uint4*>(tile + (p + k) * kCvTC + cv * V);
      const T_* e8 = reinterpret_cast<const T_*>(&u);
#pragma unroll
      for (int e = 0; e < V; ++e) f[e] = to_f32(e8[e]);
#pragma unroll
      for (int e = 0; e < V; ++e) o[e] = fmaf(wt[e][k], f[e], o[e]);
    }
#pragma unroll
    for (int e = 0; e < V; ++e) o[e] = silu_f(o[e]);
    const long long row = s_row[p + kConvK - 1];
    store_vec<T_, V>((s_pre[p + kConvK - 1] ? out_r : out_v) + row * ldo + ch, o);
  }
}

// Gated RMSNorm in place with the row held in registers: one warp per row, each lane keeps its MAXQ
// 16-byte vectors of y and z as loaded (all loads of the row in flight at once), sums (y silu(z))^2, then
// writes y silu(z) / rms * norm_w from the registers.  C / V <= 32 * MAXQ.
template <typename T_, int MAXQ>
__global__ void __launch_bounds__(256) gate_rmsnorm_reg_kernel(T_* __restrict__ y, long long ldy,
                                                               const T_* __restrict__ z, long long ldz,
                                                               const float* __restrict__ norm_w, int C,
                                                               long long rows) {
  constexpr int V = 16 / sizeof(T_);
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  const int nvec = C / V;
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    T_* yr = y + r * ldy;
    const T_* zr = z + r * ldz;
    uint4 yv[MAXQ], zv[MAXQ];
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) {
      const int v = lane + 32 * q;
      if (v < nvec) {
        yv[q] = __ldg(reinterpret_cast<const uint4*>(yr + v * V));
        zv[q] = __ldg(reinterpret_cast<const uint4*>(zr + v * V));
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) {
      if (lane + 32 * q < nvec) {
        const T_* a = reinterpret_cast<const T_*>(&yv[q]);
        const T_* c = reinterpret_cast<const T_*>(&zv[q]);
#pragma unroll
        for (int e = 0; e < V; ++e) {
          const float g = to_f32(a[e]) * silu_f(to_f32(c[e]));
          ss = fmaf(g, g, ss);
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = rsqrtf(ss / static_cast<float>(C) + kNormEps);
#pragma unroll
    for (int q = 0; q < MAXQ; ++q) {
      const int v = lane + 32 * q;
      if (v < nvec) {
        // the gated values are formed again (the same operations, so the same values) rather than held
        const T_* a = reinterpret_cast<const T_*>(&yv[q]);
        const T_* c = reinterpret_cast<const T_*>(&zv[q]);
        float o[V];
#pragma unroll
        for (int e = 0; e < V; e += 4) {
          const float4 wv = __ldg(reinterpret_cast<const float4*>(norm_w + v * V + e));
          o[e] = to_f32(a[e]) * silu_f(to_f32(c[e])) * inv * wv.x;
          o[e + 1] = to_f32(a[e + 1]) * silu_f(to_f32(c[e + 1])) * inv * wv.y;
          o[e + 2] = to_f32(a[e + 2]) * silu_f(to_f32(c[e + 2])) * inv * wv.z;
          o[e + 3] = to_f32(a[e + 3]) * silu_f(to_f32(c[e + 3])) * inv * wv.w;
        }
        store_vec<T_, V>(yr + v * V, o);
      }
    }
  }
}

// Gated RMSNorm in place, one warp per row: g = y * silu(z) over the row's C channels (C a multiple of
// V), y <- g * rsqrt(mean(g^2) + eps) * norm_w.  The second pass recomputes g from the row, which the
// first pass left in L1.
template <typename T_, int V>
__global__ void __launch_bounds__(256) gate_rmsnorm_kernel(T_* __restrict__ y, long long ldy,
                                                           const T_* __restrict__ z, long long ldz,
                                                           const float* __restrict__ norm_w, int C,
                                                           long long rows) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  const int nvec = C / V;
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    T_* yr = y + r * ldy;
    const T_* zr = z + r * ldz;
    float ss = 0.f;
    for (int v = lane; v < nvec; v += 32) {
      float a[V], c[V];
      load_vec<T_, V>(yr + v * V, a);
      load_vec<T_, V>(zr + v * V, c);
#pragma unroll
      for (int e = 0; e < V; ++e) {
        const float g = a[e] * silu_f(c[e]);
        ss = fmaf(g, g, ss);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = rsqrtf(ss / static_cast<float>(C) + kNormEps);
    for (int v = lane; v < nvec; v += 32) {
      float a[V], c[V];
      load_vec<T_, V>(yr + v * V, a);
      load_vec<T_, V>(zr + v * V, c);
#pragma unroll
      for (int e = 0; e < V; ++e) a[e] = a[e] * silu_f(c[e]) * inv * __ldg(norm_w + v * V + e);
      store_vec<T_, V>(yr + v * V, a);
    }
  }
}

}  // namespace mate
