// Chunked bidirectional selective scan (Mamba2 SSD) on tcgen05, bf16 operands, fp32 accumulation.
//
// The MA branch runs a bidirectional Mamba2 block (abstract; news article, method section) over the
// sequence S = [review tokens; video tokens in Rotary-Major-Scan order].  Per head h, with
// a_t = delta_t * A_h <= 0 and the recurrence h_t = exp(a_t) h_{t-1} + delta_t x_t B_t^T,
// y_t = h_t C_t + D_h x_t, the forward scan runs over S and the backward scan over
// [review tokens; video reversed]; the video outputs are summed.
//
// The sequence is cut into chunks of Q = 256 rows: ceil(R/Q) review chunks, then ceil(n/Q) video chunks
// (video chunk v = scan positions [vQ, vQ+Q)).  The backward scan visits the same video chunks in
// reverse order, each traversed backwards, so every video chunk holds the same tokens in both
// directions.  Inside a chunk with inclusive cumulative sums s_i = a_0 + ... + a_i and exclusive sums
// s'_i = s_i - a_i, for tokens i, j of the chunk:
//   forward  (j <= i): weight exp(s_i - s_j)     backward (j >= i): weight exp(s'_j - s'_i)
// so the two directions' intra-chunk terms add into ONE full Q x Q matrix
//   M_ij = (C_i . B_j) delta_j [ j<i: exp(s_i - s_j) | j>i: exp(s'_j - s'_i) | j=i: 2 ],
// and y_i = sum_j M_ij x_j + exp(s_i) C_i Hf^T + exp(s_last - s'_i) C_i Hb^T + 2 D_h x_i, where Hf / Hb
// are the states entering the chunk in the forward / backward traversal.  The diagonal M_ii = 2 G_ii
// delta_i usually dominates y_i; it is applied in fp32 from an fp32 copy of G_ii rather than through
// the bf16 matrix.
//
// Kernels (all exponent arguments are <= 0, so nothing overflows):
//   ssd_gram_kernel    G = C B^T per video chunk (shared by all heads: one B/C group)       [tcgen05]
//   ssd_state_kernel   chunk-local end states: Sf = sum_j exp(s_last - s_j) delta_j x_j B_j^T,
//                      Sb = sum_j exp(s'_j) delta_j x_j B_j^T, and s_last per (chunk, head)  [tcgen05]
//   ssd_carry_kernel   sequential carry over chunks: H_in(next) = exp(s_last) H_in + S     [CUDA cores]
//   ssd_output_kernel  y for one (video chunk, head): M x + row-scaled C Hf^T, C Hb^T      [tcgen05]
// Rows are gathered through the scan-order map (the permutation is done by addressing) and y is
// stored back at grid-order rows.
#pragma once
#include "common.cuh"
#include "simt.cuh"

namespace mate {

constexpr int kSsdQ = 256;   // chunk length of the tensor-core scan
constexpr int kSsdP = 64;    // head size
constexpr int kSsdN = 128;   // state size

struct SsdBf16Params {
  SeqRows s;
  int B, nh, nRc, nVc;
  const float* A_log;
  const float* Dp;
  __nv_bfloat16* Gm;  // [B][nVc][Q][Q]  C B^T of each video chunk (off-diagonal use)
  float* Gd;          // [B][nVc][Q]     its diagonal C_i . B_i in fp32
  __nv_bfloat16* Sf;  // [B][nRc + nVc][nh][N][P]   (states are stored transposed: n-major, p fastest)
  __nv_bfloat16* Sb;  // [B][nVc][nh][N][P]
  float* gl;          // [B][nRc + nVc][nh]  s_last of each chunk
  __nv_bfloat16* Hf;  // [B][nVc][nh][N][P]  state entering video chunk v, forward traversal
  __nv_bfloat16* Hb;  // [B][nVc][nh][N][P]  state entering video chunk v, backward traversal
  __nv_bfloat16* y;   // row b*y_bstride + map(q), column h*P
  int ldy;
  long long y_bstride;
};

struct RowRef {
  bool valid;
  bool video;
  long long r;
};

// Row of local index j in chunk c (review chunks first).
__device__ __forceinline__ RowRef chunk_row(const SeqRows& s, int b, int c, int nRc, int j) {
  RowRef o;
  if (c < nRc) {
    const int i = c * kSsdQ + j;
    o.valid = i < s.R;
    o.video = false;
    o.r = o.valid ? s.rrow(b, i) : 0;
  } else {
    const int q = (c - nRc) * kSsdQ + j;
    o.valid = q < s.n;
    o.video = true;
    o.r = o.valid ? s.vrow(b, q) : 0;
  }
  return o;
}

__device__ __forceinline__ const __nv_bfloat16* row_x(const SeqRows& s, const RowRef& rr) {
  return rr.video ? static_cast<const __nv_bfloat16*>(s.xv) + rr.r * s.ldxv
                  : static_cast<const __nv_bfloat16*>(s.xr) + rr.r * s.ldxr;
}
__device__ __forceinline__ const __nv_bfloat16* row_b(const SeqRows& s, const RowRef& rr) {
  return rr.video ? static_cast<const __nv_bfloat16*>(s.bv) + rr.r * s.ldbv
                  : static_cast<const __nv_bfloat16*>(s.br) + rr.r * s.ldbr;
}
__device__ __forceinline__ const __nv_bfloat16* row_c(const SeqRows& s, const RowRef& rr) {
  return rr.video ? static_cast<const __nv_bfloat16*>(s.cv) + rr.r * s.ldcv
                  : static_cast<const __nv_bfloat16*>(s.cr) + rr.r * s.ldcr;
}
__device__ __forceinline__ float row_delta(const SeqRows& s, const RowRef& rr, int h) {
  if (!rr.valid) return 0.f;
  return rr.video ? s.dv[rr.r * s.lddv + h] : s.dr[rr.r * s.lddr + h];
}

// Rows of one chunk are all review rows or all video rows, so their source arrays are CTA-uniform; the
// per-row index (through the scan-order map) is computed once per chunk into shared memory.
struct ChunkBase {
  const __nv_bfloat16* x;
  const __nv_bfloat16* b;
  const __nv_bfloat16* c;
  const float* d;
  long long ldx, ldb, ldc, ldd;
};

__device__ __forceinline__ ChunkBase chunk_base(const SeqRows& s, int c, int nRc) {
  ChunkBase o;
  if (c >= nRc) {
    o.x = static_cast<const __nv_bfloat16*>(s.xv); o.b = static_cast<const __nv_bfloat16*>(s.bv);
    o.c = static_cast<const __nv_bfloat16*>(s.cv); o.d = s.dv;
    o.ldx = s.ldxv; o.ldb = s.ldbv; o.ldc = s.ldcv; o.ldd = s.lddv;
  } else {
    o.x = static_cast<const __nv_bfloat16*>(s.xr); o.b = static_cast<const __nv_bfloat16*>(s.br);
    o.c = static_cast<const __nv_bfloat16*>(s.cr); o.d = s.dr;
    o.ldx = s.ldxr; o.ldb = s.ldbr; o.ldc = s.ldcr; o.ldd = s.lddr;
  }
  return o;
}

// srow[j] = source row of local row j of chunk c, or -1 past the end of a partial chunk.
__device__ __forceinline__ void fill_chunk_rows(const SeqRows& s, int b, int c, int nRc, long long* srow) {
  for (int j = threadIdx.x; j < kSsdQ; j += blockDim.x) {
    const RowRef rr = chunk_row(s, b, c, nRc, j);
    srow[j] = rr.valid ? rr.r : -1;
  }
}

// Inclusive prefix sum of one value per thread over the first 256 threads of the block (every thread of
// the block must call it; threads past 256 get an unused result).  warp_tot holds blockDim/32 floats.
__device__ __forceinline__ float block_scan_256(float v, float* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float u = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += u;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  float base = 0.f;
  for (int w = 0; w < warp && w < 8; ++w) base += warp_tot[w];
  __syncthreads();
  return v + base;
}

// Copy a 256-byte bf16 row (128 elements) into a K-major 128B-swizzled tile row, zero-filled if !valid.
__device__ __forceinline__ void load_row128_kmajor(uint8_t* tile, int row, const __nv_bfloat16* src, bool valid,
                                                   uint32_t kblock_bytes, int chunk) {
  cp_async16_zfill(tile + sw128_kmajor_offset(row, chunk * 8, kblock_bytes), valid ? src + chunk * 8 : src, valid);
}

// ---------------------------------------------------------------------------------------------------
// G = C B^T for one video chunk and one 128-row half of it.  grid (nVc, B, 2), 128 threads.
// ---------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128, 1) ssd_gram_kernel(const SsdBf16Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sC = smem;                // [128 i][128 n], K blocks 16 KB apart
  uint8_t* sB = smem + 32768;        // [256 j][128 n], K blocks 32 KB apart
  long long* srow = reinterpret_cast<long long*>(smem + 98304);   // [256]
  uint64_t* bar = reinterpret_cast<uint64_t*>(srow + 256);
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 1);
  const int v = blockIdx.x, b = blockIdx.y, t = blockIdx.z;
  const int c = p.nRc + v;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const ChunkBase cb = chunk_base(p.s, c, p.nRc);

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(slot, 256);
  fill_chunk_rows(p.s, b, c, p.nRc, srow);
  __syncthreads();
  for (int it = threadIdx.x; it < 128 * 16; it += 128) {
    const int r = it >> 4, ch = it & 15;
    const long long rw = srow[t * 128 + r];
    load_row128_kmajor(sC, r, cb.c + (rw < 0 ? 0 : rw) * cb.ldc, rw >= 0, 16384, ch);
  }
  for (int it = threadIdx.x; it < 256 * 16; it += 128) {
    const int r = it >> 4, ch = it & 15;
    const long long rw = srow[r];
    load_row128_kmajor(sB, r, cb.b + (rw < 0 ? 0 : rw) * cb.ldb, rw >= 0, 32768, ch);
  }
  cp_async_commit();
  cp_async_wait<0>();
  fence_proxy_async();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (threadIdx.x == 0) {
    const uint32_t idesc = idesc_bf16_f32(128, 256, 0, 0);
    const uint32_t a0 = smem_u32(sC), b0 = smem_u32(sB);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint32_t off = (s & 3) * 32;
      mma_bf16_ss(tmem, desc_sw128(a0 + (s >> 2) * 16384 + off, 16, 1024),
                  desc_sw128(b0 + (s >> 2) * 32768 + off, 16, 1024), idesc, s > 0);
    }
    mma_commit(bar);
  }
  mbar_wait(bar, 0);
  tc_fence_after();
  const int i = t * 128 + warp * 32 + lane;
  __nv_bfloat16* grow = p.Gm + ((static_cast<long long>(b) * p.nVc + v) * kSsdQ + i) * kSsdQ;
  for (int c0 = 0; c0 < 256; c0 += 32) {
    uint32_t r[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, r);
    tmem_wait_ld();
    if (c0 == (i & ~31)) {  // the diagonal element of this row lies in this slice: keep it in fp32
      float gd = 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k)
        if (k == (i & 31)) gd = __uint_as_float(r[k]);
      p.Gd[(static_cast<long long>(b) * p.nVc + v) * kSsdQ + i] = gd;
    }
    uint4* dst = reinterpret_cast<uint4*>(grow + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 pk;
      pk.x = pack_bf16x2(__uint_as_float(r[q * 8 + 0]), __uint_as_float(r[q * 8 + 1]));
      pk.y = pack_bf16x2(__uint_as_float(r[q * 8 + 2]), __uint_as_float(r[q * 8 + 3]));
      pk.z = pack_bf16x2(__uint_as_float(r[q * 8 + 4]), __uint_as_float(r[q * 8 + 5]));
      pk.w = pack_bf16x2(__uint_as_float(r[q * 8 + 6]), __uint_as_float(r[q * 8 + 7]));
      dst[q] = pk;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------------------------------
// Chunk-local end states.  grid (nRc + nVc, B, nh / heads_per_cta), 256 threads (thread j = token j).
// D[n][p] = sum_j B[j][n] * (w_j x[j][p]): A operand = the B tile read MN-major, B operand = the
// weighted x tile (MN-major), M = N_state = 128, N = P = 64, K = Q = 256.
// ---------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256, 1) ssd_state_kernel(const SsdBf16Params p, int heads_per_cta) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;                 // [256 j][128 n]
  uint8_t* sXf = smem + 65536;        // [256 j][64 p]
  uint8_t* sXb = smem + 98304;
  float* sWf = reinterpret_cast<float*>(smem + 131072);
  float* sWb = sWf + 256;
  float* wtot = sWb + 256;
  long long* srow = reinterpret_cast<long long*>(wtot + 8);   // [256]
  uint64_t* bar = reinterpret_cast<uint64_t*>(srow + 256);
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 1);
  const int c = blockIdx.x, b = blockIdx.y;
  const ChunkBase cb = chunk_base(p.s, c, p.nRc);
  const bool video = c >= p.nRc;
  const int nC = p.nRc + p.nVc;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = threadIdx.x;

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(slot, 128);
  fill_chunk_rows(p.s, b, c, p.nRc, srow);
  __syncthreads();
  for (int it = threadIdx.x; it < 256 * 16; it += 256) {
    const int r = it >> 4, ch = it & 15;
    const long long rw = srow[r];
    load_row128_kmajor(sB, r, cb.b + (rw < 0 ? 0 : rw) * cb.ldb, rw >= 0, 32768, ch);
  }
  cp_async_commit();
  const long long myrw = srow[j];
  tc_fence_after();
  const uint32_t tmem = *slot;
  uint32_t phase = 0;

  // x rows of this thread's 8 items (row it>>3, 16-byte chunk it&7); the next head's rows are fetched
  // while the current head's MMAs run
  uint4 xr[8];
  auto load_x = [&](int h) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int it = threadIdx.x + u * 256;
      const long long rw = srow[it >> 3];
      xr[u] = rw >= 0 ? __ldg(reinterpret_cast<const uint4*>(cb.x + rw * cb.ldx + h * kSsdP + (it & 7) * 8))
                      : make_uint4(0, 0, 0, 0);
    }
  };
  load_x(blockIdx.z * heads_per_cta);
  float dl_next = myrw >= 0 ? cb.d[myrw * cb.ldd + blockIdx.z * heads_per_cta] : 0.f;

  for (int hh = 0; hh < heads_per_cta; ++hh) {
    const int h = blockIdx.z * heads_per_cta + hh;
    const float A = -__expf(p.A_log[h]);
    const float dl = dl_next;
    const float a = dl * A;
    const float s = block_scan_256(a, wtot);
    if (j == 255) wtot[8 - 1] = s;  // reuse slot 7 for s_last after the scan finished with wtot
    __syncthreads();
    const float s_last = wtot[7];
    sWf[j] = __expf(s_last - s) * dl;
    sWb[j] = __expf(s - a) * dl;
    __syncthreads();
    // weighted x tiles, 8 bf16 (one 16-byte chunk) per item; 8 items per row
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int it = threadIdx.x + u * 256;
      const int r = it >> 3, ch = it & 7;
      const float wf = sWf[r], wb = sWb[r];
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xr[u]);
      uint4 of, ob;
      uint32_t* pf = reinterpret_cast<uint32_t*>(&of);
      uint32_t* pb = reinterpret_cast<uint32_t*>(&ob);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack_bf16x2(xw[e]);
        pf[e] = pack_bf16x2(f.x * wf, f.y * wf);
        pb[e] = pack_bf16x2(f.x * wb, f.y * wb);
      }
      const uint32_t off = sw128_mnmajor_offset(r, ch * 8, 32768);
      *reinterpret_cast<uint4*>(sXf + off) = of;
      *reinterpret_cast<uint4*>(sXb + off) = ob;
    }
    if (hh == 0) cp_async_wait<0>();
    fence_proxy_async();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16_f32(128, 64, 1, 1);
      const uint32_t ab = smem_u32(sB), xf = smem_u32(sXf), xb = smem_u32(sXb);
#pragma unroll 4
      for (int k = 0; k < 16; ++k) {
        const uint64_t ad = desc_sw128(ab + k * 2048, 32768, 1024);
        mma_bf16_ss(tmem, ad, desc_sw128(xf + k * 2048, 32768, 1024), idesc, k > 0);
        if (video) mma_bf16_ss(tmem + 64, ad, desc_sw128(xb + k * 2048, 32768, 1024), idesc, k > 0);
      }
      mma_commit(bar);
    }
    if (hh + 1 < heads_per_cta) {
      load_x(h + 1);
      dl_next = myrw >= 0 ? cb.d[myrw * cb.ldd + h + 1] : 0.f;
    }
    mbar_wait(bar, phase);
    phase ^= 1;
    tc_fence_after();
    const int dir = warp >> 2, quad = warp & 3;
    const int nidx = quad * 32 + lane;
    if (dir == 0 || video) {
      __nv_bfloat16* dst = dir == 0
          ? p.Sf + ((static_cast<long long>(b) * nC + c) * p.nh + h) * (kSsdP * kSsdN)
          : p.Sb + ((static_cast<long long>(b) * p.nVc + (c - p.nRc)) * p.nh + h) * (kSsdP * kSsdN);
      // lane = state row n: its 64 p values are one contiguous 128-byte row of the [N][P] state
      for (int pc = 0; pc < 2; ++pc) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + dir * 64 + pc * 32, r);
        tmem_wait_ld();
        uint4* d4 = reinterpret_cast<uint4*>(dst + nidx * kSsdP + pc * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 pk;
          pk.x = pack_bf16x2(__uint_as_float(r[q * 8 + 0]), __uint_as_float(r[q * 8 + 1]));
          pk.y = pack_bf16x2(__uint_as_float(r[q * 8 + 2]), __uint_as_float(r[q * 8 + 3]));
          pk.z = pack_bf16x2(__uint_as_float(r[q * 8 + 4]), __uint_as_float(r[q * 8 + 5]));
          pk.w = pack_bf16x2(__uint_as_float(r[q * 8 + 6]), __uint_as_float(r[q * 8 + 7]));
          d4[q] = pk;
        }
      }
    }
    if (threadIdx.x == 0) p.gl[(static_cast<long long>(b) * nC + c) * p.nh + h] = s_last;
    tc_fence_before();
    __syncthreads();
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ---------------------------------------------------------------------------------------------------
// Sequential carry across chunks.  grid (P*N/8/128, nh, 2*B), 128 threads; thread = 8 state elements.
// Review chunks are visited first (same order in both directions); then the video chunks ascending
// (forward) or descending (backward).  Writes the state entering each video chunk.
// ---------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128) ssd_carry_kernel(const SsdBf16Params p) {
  const int e8 = blockIdx.x * blockDim.x + threadIdx.x;  // vector of 8 elements
  const int h = blockIdx.y;
  const int dir = blockIdx.z & 1, b = blockIdx.z >> 1;
  const int nC = p.nRc + p.nVc;
  constexpr int PN = kSsdP * kSsdN;
  if (e8 * 8 >= PN) return;
  float H[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) H[e] = 0.f;
  auto step = [&](float glv, uint4 sv) {
    const float g = __expf(glv);
    const uint32_t* u = reinterpret_cast<const uint32_t*>(&sv);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(u[e]);
      H[2 * e] = fmaf(g, H[2 * e], f.x);
      H[2 * e + 1] = fmaf(g, H[2 * e + 1], f.y);
    }
  };
  auto store = [&](__nv_bfloat16* base) {
    uint4 o;
    uint32_t* u = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) u[e] = pack_bf16x2(H[2 * e], H[2 * e + 1]);
    *reinterpret_cast<uint4*>(base + e8 * 8) = o;
  };
  for (int c = 0; c < p.nRc; ++c) {
    const long long ci = (static_cast<long long>(b) * nC + c) * p.nh + h;
    step(p.gl[ci], __ldg(reinterpret_cast<const uint4*>(p.Sf + ci * PN) + e8));
  }
  constexpr int U = 4;
  for (int k0 = 0; k0 < p.nVc; k0 += U) {
    uint4 sv[U];
    float gv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + u;
      if (k < p.nVc) {
        const int v = dir == 0 ? k : p.nVc - 1 - k;
        const long long ci = (static_cast<long long>(b) * nC + p.nRc + v) * p.nh + h;
        const long long vi = (static_cast<long long>(b) * p.nVc + v) * p.nh + h;
        gv[u] = p.gl[ci];
        sv[u] = __ldg(reinterpret_cast<const uint4*>((dir == 0 ? p.Sf + ci * PN : p.Sb + vi * PN)) + e8);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + u;
      if (k < p.nVc) {
        const int v = dir == 0 ? k : p.nVc - 1 - k;
        const long long vi = (static_cast<long long>(b) * p.nVc + v) * p.nh + h;
        store((dir == 0 ? p.Hf : p.Hb) + vi * PN);
        step(gv[u], sv[u]);
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------------
// Outputs of the video chunks: persistent, warp-specialised.  One work item = (sample, video chunk, head,
// 128-row tile t of the chunk); a CTA walks items blockIdx.x, blockIdx.x + gridDim.x, ...
//
//   warps 0..3   loaders: gather the item's x rows (all 256, MN-major) and the C rows of the tile
//                (K-major) with TMA four-row gathers (tile::gather4), load the incoming states Hf / Hb
//                (MN-major) with 2D TMA, into one of two shared-memory buffers; compute the cumulative
//                sums and the decay factor tables of the item.
//   warps 4..11  transform (two warps per TMEM lane quadrant, alternating 8-column chunks): read the
//                tile's 128 rows of G = C B^T (bf16, global/L2), form
//                M_ij = G_ij delta_j dec(i, j) (diagonal excluded) and store M straight into TMEM as
//                the A operand of the next MMA (two bf16 per 32-bit column).
//   MMA issue    lane 0 of warp 4, once all transform warps stored M: Yd = M x (A from TMEM),
//                Yf = C Hf^T, Yb = C Hb^T into one of two TMEM accumulator sets.  (16 warps in total: a
//                17th warp would put 5 warps on one SM sub-partition, beyond its register file.)
//   warps 12..15 epilogue: y_i = Yd + exp(s_i) Yf + exp(s_last - s'_i) Yb + 2 (D + G_ii delta_i) x_i,
//                stored at the grid-order row of the token.
//
// Decay factors: for a 64-row block ib and a column j of an EARLIER 64-block (forward direction), the
// reference k = 64 ib - 1 lies between them, so exp(s_i - s_j) = exp(s_i - s_k) exp(s_k - s_j) (both
// exponents <= 0): a per-row factor times a per-(ib, j) column factor.  Columns of LATER blocks use
// k' = 64 (ib + 1) with the exclusive sums.  Only the 64 x 64 diagonal blocks need one exponential per
// element.
// TMEM columns: [0, 128) M; accumulator set a at 128 + 192 a: Yd [+0, +64), Yf [+64, +128), Yb [+128, +192).
// ---------------------------------------------------------------------------------------------------
constexpr int kOutLoadWarps = 4, kOutXformWarps = 8, kOutEpiWarps = 4;
constexpr int kOutMmaWarp = kOutLoadWarps;                                    // issues from its lane 0
constexpr int kSsdOutThreads = (kOutLoadWarps + kOutXformWarps + kOutEpiWarps) * 32;   // 512
constexpr uint32_t kOutBuf = 108544;                                         // bytes per operand buffer
constexpr uint32_t kOutOffC = 32768, kOutOffHf = 65536, kOutOffHb = 81920, kOutOffTbl = 98304;
constexpr uint32_t kOutSmem = 2 * kOutBuf + 256;

// Tensor maps of the output kernel: x and C rows of the video arrays (one-row boxes of 64 columns, for
// four-row gathers) and the carried states ([N rows][P] per chunk and head, 64 x 128 boxes).
struct SsdOutMaps {
  CUtensorMap x, c, hf, hb;
  int rows;   // row extent of the x / C maps; gathers of invalid rows use this (out of range -> zeros)
};

struct OutTables {   // per buffer, at kOutOffTbl
  float sdl[256], ss[256], ssx[256];
  float uf[128], ub[128];       // per tile row
  float wf[2][256], wb[2][256]; // per 64-row block of the tile (ib = 2t + q)
  int srow[256];                // source row of each chunk row (-1 past the end of a partial chunk)
  float wtot[4];
};

__global__ void __launch_bounds__(kSsdOutThreads, 1) ssd_output_kernel(const SsdBf16Params p,
                                                                        const __grid_constant__ SsdOutMaps mp) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * kOutBuf);
  uint64_t* ld_full = bars;        // [2] loaders -> consumers (count 128)
  uint64_t* ld_empty = bars + 2;   // [2] MMA commit + epilogue warps -> loaders (count 5)
  uint64_t* m_full = bars + 4;     // [2] per K half of M: transform -> MMA (count 256)
  uint64_t* m_empty = bars + 6;    // [2] per K half of M: MMA commit -> transform (count 1)
  uint64_t* y_full = bars + 8;     // [2] MMA commit -> epilogue (count 1)
  uint64_t* y_empty = bars + 10;   // [2] epilogue warps -> MMA (count 4)
  uint32_t* slot = reinterpret_cast<uint32_t*>(bars + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nitems = p.B * p.nVc * p.nh * 2;

  if (threadIdx.x == 0) {
    for (int q = 0; q < 2; ++q) {
      mbar_init(&ld_full[q], 129);   // 128 loader threads + the byte-count arrival
      mbar_init(&ld_empty[q], 5);
      mbar_init(&y_full[q], 1);
      mbar_init(&y_empty[q], 4);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&m_full[q], 256);
      mbar_init(&m_empty[q], 1);
    }
    mbar_fence_init();
  }
  if (warp == kOutMmaWarp) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;

  auto decode = [&](int it, int& b, int& v, int& h, int& t) {
    t = it & 1;
    int rest = it >> 1;
    h = rest % p.nh;
    rest /= p.nh;
    v = rest % p.nVc;
    b = rest / p.nVc;
  };

  if (warp < kOutLoadWarps) {
    // ------------------------------------------------------------------------------ loaders
    const int lt = threadIdx.x;  // 0..127
    int k = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++k) {
      const int buf = k & 1, use = k >> 1;
      if (!mbar_wait(&ld_empty[buf], (use & 1) ^ 1)) break;
      int b, v, h, t;
      decode(it, b, v, h, t);
      const int c = p.nRc + v;
      const ChunkBase cb = chunk_base(p.s, c, p.nRc);
      uint8_t* B0 = smem + buf * kOutBuf;
      OutTables& tb = *reinterpret_cast<OutTables*>(B0 + kOutOffTbl);
      for (int j = lt; j < 256; j += 128) {
        const RowRef rr = chunk_row(p.s, b, c, p.nRc, j);
        tb.srow[j] = rr.valid ? static_cast<int>(rr.r) : -1;
      }
      if (lt == 0) mbar_arrive_expect_tx(&ld_full[buf], 3 * 32768);   // x (32 KB), C (32 KB), Hf + Hb (32 KB)
      named_bar_sync(1, 128);
      // TMA: x rows (all 256, 4 per gather), C rows of the tile (2 column blocks), the two states
      auto rowid = [&](int j) { const int rw = tb.srow[j]; return rw < 0 ? mp.rows : rw; };
      if (lt < 64) {
        const int g = lt;
        tma_gather4(&mp.x, &ld_full[buf], B0 + g * 512, h * kSsdP, rowid(4 * g), rowid(4 * g + 1), rowid(4 * g + 2),
                    rowid(4 * g + 3));
      } else {
        const int g = (lt - 64) & 31, kb = (lt - 64) >> 5;
        const int j = t * 128 + 4 * g;
        tma_gather4(&mp.c, &ld_full[buf], B0 + kOutOffC + kb * 16384 + g * 512, kb * 64, rowid(j), rowid(j + 1),
                    rowid(j + 2), rowid(j + 3));
      }
      if (lt == 0) {
        const int hrow = static_cast<int>(((static_cast<long long>(b) * p.nVc + v) * p.nh + h) * kSsdN);
        tma_load_2d(&mp.hf, &ld_full[buf], B0 + kOutOffHf, 0, hrow);
        tma_load_2d(&mp.hb, &ld_full[buf], B0 + kOutOffHb, 0, hrow);
      }
      // cumulative sums: thread lt owns rows 2 lt and 2 lt + 1
      const float A = -__expf(p.A_log[h]);
      float dl[2], a[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int rw = tb.srow[2 * lt + e];
        dl[e] = rw >= 0 ? cb.d[static_cast<long long>(rw) * cb.ldd + h] : 0.f;
        a[e] = dl[e] * A;
      }
      float incl = a[0] + a[1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float u2 = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += u2;
      }
      if (lane == 31) tb.wtot[warp] = incl;
      named_bar_sync(1, 128);
      for (int w = 0; w < warp; ++w) incl += tb.wtot[w];
      const float s1 = incl, s0 = incl - a[1];
      tb.sdl[2 * lt] = dl[0];
      tb.sdl[2 * lt + 1] = dl[1];
      tb.ss[2 * lt] = s0;
      tb.ss[2 * lt + 1] = s1;
      tb.ssx[2 * lt] = s0 - a[0];
      tb.ssx[2 * lt + 1] = s1 - a[1];
      named_bar_sync(1, 128);
      {
        const int i = t * 128 + lt, ib = i >> 6;
        tb.uf[lt] = ib > 0 ? __expf(tb.ss[i] - tb.ss[64 * ib - 1]) : 0.f;
        tb.ub[lt] = ib < 3 ? __expf(tb.ssx[64 * ib + 64] - tb.ssx[i]) : 0.f;
      }
      for (int j = lt; j < 256; j += 128) {
        const float dj = tb.sdl[j], sj = tb.ss[j], sxj = tb.ssx[j];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int ib = 2 * t + q;
          tb.wf[q][j] = (ib > 0 && j < 64 * ib) ? dj * __expf(tb.ss[64 * ib - 1] - sj) : 0.f;
          tb.wb[q][j] = (ib < 3 && j >= 64 * ib + 64) ? dj * __expf(sxj - tb.ssx[64 * ib + 64]) : 0.f;
        }
      }
      mbar_arrive(&ld_full[buf]);
    }
  } else if (warp < kOutLoadWarps + kOutXformWarps) {
    // ------------------------------------------------------------------------------ transform
    const int xw = warp - kOutLoadWarps;
    const int quad = warp & 3, half = xw >> 2;
    const int r = quad * 32 + lane;
    int k = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++k) {
      const int buf = k & 1, use = k >> 1;
      int b, v, h, t;
      decode(it, b, v, h, t);
      const int i = t * 128 + r, ib = i >> 6;
      // the two warps of a lane quadrant take alternating 8-column chunks of the row, so both get half of
      // the diagonal block's exponentials
      const __nv_bfloat16* grow = p.Gm + ((static_cast<long long>(b) * p.nVc + v) * kSsdQ + i) * kSsdQ + half * 8;
      // the row's 16 chunks of G (8 bf16 each, 256 bytes) are all in flight before the waits and are
      // consumed in order through a shifting register window (keeps the chunk loop rolled: the four roles'
      // code must share the instruction cache)
      const uint4* gsrc = reinterpret_cast<const uint4*>(grow);
      uint4 gw[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) gw[q] = __ldg(gsrc + 2 * q);
      if (!mbar_wait(&ld_full[buf], use & 1)) break;
      const OutTables& tb = *reinterpret_cast<const OutTables*>(smem + buf * kOutBuf + kOutOffTbl);
      const float ufi = tb.uf[r], ubi = tb.ub[r], si = tb.ss[i], sxi = tb.ssx[i];
      const float* wfr = tb.wf[ib - 2 * t];
      const float* wbr = tb.wb[ib - 2 * t];
      const uint32_t tm_row = tmem + (static_cast<uint32_t>(quad * 32) << 16) + half * 4;
      const int acc = k & 1;
      bool ok = true, mma_ok = true;
      // M is produced and consumed in two K halves (TMEM columns [0, 64) and [64, 128)): the MMAs of the
      // first half run while the second half is being formed
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        if (!mbar_wait(&m_empty[hh], (k & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int q = 8 * hh; q < 8 * hh + 8; ++q) {
          const uint4 gc = gw[0];
#pragma unroll
          for (int z = 0; z < 15; ++z) gw[z] = gw[z + 1];
          const int j0 = (2 * q + half) * 8;
          const int jb = j0 >> 6;   // same for the whole warp (all lanes are rows of one 64-block)
          const uint32_t* gu = reinterpret_cast<const uint32_t*>(&gc);
          uint32_t pk[4];
          if (jb != ib) {
            const float u = jb < ib ? ufi : ubi;
            const float* w = (jb < ib ? wfr : wbr) + j0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 gf = unpack_bf16x2(gu[e]);
              const float2 w2 = *reinterpret_cast<const float2*>(w + 2 * e);
              pk[e] = pack_bf16x2(gf.x * (u * w2.x), gf.y * (u * w2.y));
            }
          } else {
            // one exponential per element: forward weight below the diagonal, backward above; the
            // diagonal itself is added in fp32 in the epilogue
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int jj = j0 + 2 * e;
              const float2 gf = unpack_bf16x2(gu[e]);
              const float2 sj = *reinterpret_cast<const float2*>(tb.ss + jj);
              const float2 xj = *reinterpret_cast<const float2*>(tb.ssx + jj);
              const float2 dj = *reinterpret_cast<const float2*>(tb.sdl + jj);
              const float f0 = jj == i ? 0.f : dj.x * __expf(jj < i ? si - sj.x : xj.x - sxi);
              const float f1 = jj + 1 == i ? 0.f : dj.y * __expf(jj + 1 < i ? si - sj.y : xj.y - sxi);
              pk[e] = pack_bf16x2(gf.x * f0, gf.y * f1);
            }
          }
          tmem_st4(tm_row + q * 8, pk[0], pk[1], pk[2], pk[3]);   // columns of chunk 2q + half
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&m_full[hh]);
        if (warp == kOutMmaWarp) {
          if (lane == 0) {
            // -------------------------------------------------------------------- MMA issue
            const uint32_t idesc = idesc_bf16_f32(128, 64, 0, 1);
            if (hh == 0) mma_ok = mbar_wait(&y_empty[acc], (use & 1) ^ 1);
            mma_ok = mma_ok && mbar_wait(&m_full[hh], k & 1);
            if (mma_ok) {
              tc_fence_after();
              const uint32_t b0 = smem_u32(smem + buf * kOutBuf);
              const uint32_t ybase = tmem + 128 + acc * 192;
#pragma unroll
              for (int q = 8 * hh; q < 8 * hh + 8; ++q)   // Yd = M x (M in TMEM, 8 columns per 16 elements)
                mma_bf16_ts(ybase, tmem + q * 8, desc_sw128(b0 + q * 2048, 32768, 1024), idesc, q > 0);
              mma_commit(&m_empty[hh]);
              if (hh == 1) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {  // Yf = C Hf^T, Yb = C Hb^T, K = N = 128
                  const uint64_t ad = desc_sw128(b0 + kOutOffC + (q >> 2) * 16384 + (q & 3) * 32, 16, 1024);
                  mma_bf16_ss(ybase + 64, ad, desc_sw128(b0 + kOutOffHf + q * 2048, 16384, 1024), idesc, q > 0);
                  mma_bf16_ss(ybase + 128, ad, desc_sw128(b0 + kOutOffHb + q * 2048, 16384, 1024), idesc, q > 0);
                }
                mma_commit(&y_full[acc]);
                mma_commit(&ld_empty[buf]);
              }
            }
          }
          __syncwarp();
        }
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    int k = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++k) {
      const int buf = k & 1, acc = k & 1, use = k >> 1;
      int b, v, h, t;
      decode(it, b, v, h, t);
      if (!mbar_wait(&y_full[acc], use & 1)) break;
      tc_fence_after();
      const uint8_t* B0 = smem + buf * kOutBuf;
      const OutTables& tb = *reinterpret_cast<const OutTables*>(B0 + kOutOffTbl);
      const int i = t * 128 + r;
      const int len = min(kSsdQ, p.s.n - v * kSsdQ);
      const bool ok = i < len;
      const float si = tb.ss[i], sxi = tb.ssx[i], slast = tb.ss[255], dli = tb.sdl[i];
      // x row of this token (packed bf16 pairs) for the skip and diagonal terms
      uint32_t xw[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 xv = *reinterpret_cast<const uint4*>(B0 + sw128_mnmajor_offset(i, q * 8, 32768));
        xw[q * 4 + 0] = xv.x; xw[q * 4 + 1] = xv.y; xw[q * 4 + 2] = xv.z; xw[q * 4 + 3] = xv.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ld_empty[buf]);
      const float ef = __expf(si);
      const float eb = __expf(slast - sxi);
      const float D2 = 2.f * (p.Dp[h] + (ok ? p.Gd[(static_cast<long long>(b) * p.nVc + v) * kSsdQ + i] * dli : 0.f));
      __nv_bfloat16* yrow = p.y + (b * p.y_bstride + p.s.map(v * kSsdQ + (ok ? i : 0))) * p.ldy + h * kSsdP;
      const uint32_t ybase = tmem + (static_cast<uint32_t>(quad * 32) << 16) + 128 + acc * 192;
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {   // 16 columns at a time
        uint32_t yd[16], yf[16], yb[16];
        tmem_ld16(ybase + pc * 16, yd);
        tmem_ld16(ybase + 64 + pc * 16, yf);
        tmem_ld16(ybase + 128 + pc * 16, yb);
        tmem_wait_ld();
        if (ok) {
          uint32_t ou[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 xf = unpack_bf16x2(xw[pc * 8 + e]);
            const int k0 = 2 * e;
            const float y0 = __uint_as_float(yd[k0]) + ef * __uint_as_float(yf[k0]) + eb * __uint_as_float(yb[k0]) + D2 * xf.x;
            const float y1 = __uint_as_float(yd[k0 + 1]) + ef * __uint_as_float(yf[k0 + 1]) +
                             eb * __uint_as_float(yb[k0 + 1]) + D2 * xf.y;
            ou[e] = pack_bf16x2(y0, y1);
          }
          uint4* dst = reinterpret_cast<uint4*>(yrow + pc * 16);
          dst[0] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
          dst[1] = make_uint4(ou[4], ou[5], ou[6], ou[7]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&y_empty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kOutMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mate
