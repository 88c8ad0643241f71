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
// Outputs of one video chunk and head.  grid (nVc, B, nh), 256 threads (8 warps).
//
// The Q x Q coefficient matrix M_ij = G_ij delta_j dec(i, j) is built one 128-row tile at a time in
// shared memory (bf16, K-major) from the bf16 G of the chunk.  The decay factors are exact products of
// cumulative-sum exponentials; only the 64 x 64 diagonal blocks need one exponential per element.  For a
// 64-row block ib and a column j of an EARLIER block (forward direction, j < i) the reference index
// k = 64 ib - 1 lies between them, so
//     exp(s_i - s_j) = exp(s_i - s_k) * exp(s_k - s_j)      (both exponents <= 0),
// a per-row factor times a per-(ib, j) column factor.  Columns of LATER blocks (backward direction) use
// k' = 64 (ib + 1):  exp(s'_j - s'_i) = exp(s'_j - s'_k') * exp(s'_k' - s'_i).
// TMEM columns: [t*64, +64) sum_j M_ij x_j for row tile t; [128 + t*64, +64) C Hf^T; [256 + t*64, +64)
// C Hb^T.
// ---------------------------------------------------------------------------------------------------
constexpr int kSsdOutThreads = 512;

__global__ void __launch_bounds__(kSsdOutThreads, 1) ssd_output_kernel(const SsdBf16Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sM = smem;                 // [128 i][256 j] K-major, K blocks 16 KB apart (G tile, then M tile)
  uint8_t* sX = smem + 65536;         // [256 j][64 p] MN-major
  uint8_t* sC = smem + 98304;         // [256 i][128 n] K-major, K blocks 32 KB apart
  uint8_t* sHf = smem + 163840;       // [128 n][64 p] MN-major (B operand of C H^T with K = n)
  uint8_t* sHb = smem + 180224;
  float* sdl = reinterpret_cast<float*>(smem + 196608);
  float* ss = sdl + 256;              // inclusive cumulative sums s_i
  float* ssx = ss + 256;              // exclusive sums s'_i = s_i - a_i
  float* uf = ssx + 256;              // per-row forward factor exp(s_i - s_{64 ib - 1})
  float* ub = uf + 256;               // per-row backward factor exp(s'_{64 ib + 64} - s'_i)
  float* wf = ub + 256;               // [4][256] delta_j exp(s_{64 ib - 1} - s_j), j < 64 ib
  float* wb = wf + 1024;              // [4][256] delta_j exp(s'_j - s'_{64 ib + 64}), j >= 64 ib + 64
  float* wtot = wb + 1024;            // [16]
  long long* srow = reinterpret_cast<long long*>(wtot + 16);   // [256]
  uint64_t* bar = reinterpret_cast<uint64_t*>(srow + 256);
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 1);
  const int v = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
  const int c = p.nRc + v;
  const ChunkBase cb = chunk_base(p.s, c, p.nRc);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  constexpr int PN = kSsdP * kSsdN;
  constexpr int NT = kSsdOutThreads;

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(slot, 512);
  fill_chunk_rows(p.s, b, c, p.nRc, srow);
  const __nv_bfloat16* gbase = p.Gm + (static_cast<long long>(b) * p.nVc + v) * kSsdQ * kSsdQ;
  // G rows 0..127 straight into the M tile (transformed in place below)
  for (int it = tid; it < 128 * 32; it += NT) {
    const int r = it >> 5, cc = it & 31;
    cp_async16(sM + sw128_kmajor_offset(r, cc * 8, 16384), gbase + r * kSsdQ + cc * 8);
  }
  __syncthreads();  // srow
  for (int it = tid; it < 256 * 8; it += NT) {
    const int r = it >> 3, ch = it & 7;
    const long long rw = srow[r];
    cp_async16_zfill(sX + sw128_mnmajor_offset(r, ch * 8, 32768), cb.x + (rw < 0 ? 0 : rw) * cb.ldx + h * kSsdP + ch * 8,
                     rw >= 0);
  }
  for (int it = tid; it < 256 * 16; it += NT) {
    const int r = it >> 4, ch = it & 15;
    const long long rw = srow[r];
    load_row128_kmajor(sC, r, cb.c + (rw < 0 ? 0 : rw) * cb.ldc, rw >= 0, 32768, ch);
  }
  const long long vi = (static_cast<long long>(b) * p.nVc + v) * p.nh + h;
  for (int it = tid; it < 128 * 8; it += NT) {
    const int r = it >> 3, ch = it & 7;
    cp_async16(sHf + sw128_mnmajor_offset(r, ch * 8, 16384), p.Hf + vi * PN + r * kSsdP + ch * 8);
    cp_async16(sHb + sw128_mnmajor_offset(r, ch * 8, 16384), p.Hb + vi * PN + r * kSsdP + ch * 8);
  }
  cp_async_commit();

  // cumulative sums and decay factor tables (threads 0..255 = chunk rows)
  const int j = tid & 255;
  const bool data = tid < 256;
  const long long myrw = srow[j];
  const int len = min(kSsdQ, p.s.n - v * kSsdQ);
  const float A = -__expf(p.A_log[h]);
  const float dl = (data && myrw >= 0) ? cb.d[myrw * cb.ldd + h] : 0.f;
  const float a = dl * A;
  const float s = block_scan_256(a, wtot);
  if (data) {
    sdl[j] = dl;
    ss[j] = s;
    ssx[j] = s - a;
  }
  __syncthreads();
  if (data) {
    const int ib = j >> 6;
    uf[j] = ib > 0 ? __expf(s - ss[64 * ib - 1]) : 0.f;
    ub[j] = ib < 3 ? __expf(ssx[64 * ib + 64] - (s - a)) : 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      wf[q * 256 + j] = (q > 0 && j < 64 * q) ? dl * __expf(ss[64 * q - 1] - s) : 0.f;
      wb[q * 256 + j] = (q < 3 && j >= 64 * q + 64) ? dl * __expf((s - a) - ssx[64 * q + 64]) : 0.f;
    }
  }
  cp_async_wait<0>();
  fence_proxy_async();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;

  if (tid == 0) {
    const uint32_t idesc = idesc_bf16_f32(128, 64, 0, 1);
    const uint32_t c0 = smem_u32(sC), hf = smem_u32(sHf), hb = smem_u32(sHb);
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t off = (k & 3) * 32;
        const uint64_t ad = desc_sw128(c0 + (k >> 2) * 32768 + t * 16384 + off, 16, 1024);
        mma_bf16_ss(tmem + 128 + t * 64, ad, desc_sw128(hf + k * 2048, 16384, 1024), idesc, k > 0);
        mma_bf16_ss(tmem + 256 + t * 64, ad, desc_sw128(hb + k * 2048, 16384, 1024), idesc, k > 0);
      }
  }

  // build mapping: thread -> one row of the tile (lanes = consecutive rows: conflict-free swizzled
  // accesses, broadcast column tables) and every fourth 16-byte column chunk
  const int r = (warp & 3) * 32 + lane;
  const int cg = warp >> 2;
  // scale 8 G values of row i, columns j0..j0+7 (one 64-block) into M values
  auto transform = [&](uint4 g8, int i, int j0) -> uint4 {
    const int ib = i >> 6, jb = j0 >> 6;
    const uint32_t* gu = reinterpret_cast<const uint32_t*>(&g8);
    uint4 o;
    uint32_t* ou = reinterpret_cast<uint32_t*>(&o);
    if (jb != ib) {
      const float u = jb < ib ? uf[i] : ub[i];
      const float4* w4 = reinterpret_cast<const float4*>((jb < ib ? wf : wb) + ib * 256 + j0);
      const float4 wa = w4[0], wc = w4[1];
      const float w[8] = {wa.x, wa.y, wa.z, wa.w, wc.x, wc.y, wc.z, wc.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 g = unpack_bf16x2(gu[e]);
        ou[e] = pack_bf16x2(g.x * u * w[2 * e], g.y * u * w[2 * e + 1]);
      }
    } else {
      const float si = ss[i], sxi = ssx[i];
      const float4* s4 = reinterpret_cast<const float4*>(ss + j0);
      const float4* x4 = reinterpret_cast<const float4*>(ssx + j0);
      const float4* d4 = reinterpret_cast<const float4*>(sdl + j0);
      const float4 sa = s4[0], sb = s4[1], xa = x4[0], xb = x4[1], da = d4[0], db = d4[1];
      const float sj[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
      const float xj[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
      const float dj[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 g = unpack_bf16x2(gu[e]);
        float m2[2];
#pragma unroll
        for (int z = 0; z < 2; ++z) {
          const int k = 2 * e + z, jj = j0 + k;
          // the diagonal (j = i) is added in fp32 in the epilogue
          const float dec = jj < i ? __expf(si - sj[k]) : (jj > i ? __expf(xj[k] - sxi) : 0.f);
          m2[z] = (z == 0 ? g.x : g.y) * dj[k] * dec;
        }
        ou[e] = pack_bf16x2(m2[0], m2[1]);
      }
    }
    return o;
  };

  // row tile 0: G already in sM, transform in place
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int cc = cg + 4 * k;
    uint4* loc = reinterpret_cast<uint4*>(sM + sw128_kmajor_offset(r, cc * 8, 16384));
    *loc = transform(*loc, r, cc * 8);
  }
  fence_proxy_async();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16_f32(128, 64, 0, 1);
    const uint32_t m0 = smem_u32(sM), x0 = smem_u32(sX);
#pragma unroll 4
    for (int k = 0; k < 16; ++k)
      mma_bf16_ss(tmem, desc_sw128(m0 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                  desc_sw128(x0 + k * 2048, 32768, 1024), idesc, k > 0);
    mma_commit(bar);
  }
  // row tile 1: G rows 128..255 fetched into registers while tile 0 multiplies
  uint4 g1[8];
#pragma unroll
  for (int k = 0; k < 8; ++k)
    g1[k] = __ldg(reinterpret_cast<const uint4*>(gbase + (128 + r) * kSsdQ + (cg + 4 * k) * 8));
  mbar_wait(bar, 0);
  tc_fence_after();
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int cc = cg + 4 * k;
    *reinterpret_cast<uint4*>(sM + sw128_kmajor_offset(r, cc * 8, 16384)) = transform(g1[k], 128 + r, cc * 8);
  }
  fence_proxy_async();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16_f32(128, 64, 0, 1);
    const uint32_t m0 = smem_u32(sM), x0 = smem_u32(sX);
#pragma unroll 4
    for (int k = 0; k < 16; ++k)
      mma_bf16_ss(tmem + 64, desc_sw128(m0 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                  desc_sw128(x0 + k * 2048, 32768, 1024), idesc, k > 0);
    mma_commit(bar);
  }
  mbar_wait(bar, 1);
  tc_fence_after();

  // epilogue: warp w -> TMEM lane quadrant w%4, row tile (w/4)%2, 32-column half w/8
  const int quad = warp & 3, t = (warp >> 2) & 1, pc = warp >> 3;
  const int i = t * 128 + quad * 32 + lane;
  const bool ok = i < len;
  const float ef = __expf(ss[i]);
  const float eb = __expf(ss[255] - ssx[i]);
  // diagonal of both directions (weight 1 each) plus the two skip terms, in fp32
  const float D2 = 2.f * (p.Dp[h] + (ok ? p.Gd[(static_cast<long long>(b) * p.nVc + v) * kSsdQ + i] * sdl[i] : 0.f));
  __nv_bfloat16* yrow = p.y + (b * p.y_bstride + p.s.map(v * kSsdQ + (ok ? i : 0))) * p.ldy + h * kSsdP;
  const uint32_t lanebase = static_cast<uint32_t>(quad * 32) << 16;
  {
    uint32_t yd[32], yf[32], yb[32];
    tmem_ld32(tmem + lanebase + t * 64 + pc * 32, yd);
    tmem_ld32(tmem + lanebase + 128 + t * 64 + pc * 32, yf);
    tmem_ld32(tmem + lanebase + 256 + t * 64 + pc * 32, yb);
    tmem_wait_ld();
    if (ok) {
      uint4 out[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 xv = *reinterpret_cast<const uint4*>(sX + sw128_mnmajor_offset(i, pc * 32 + q * 8, 32768));
        const uint32_t* xu = reinterpret_cast<const uint32_t*>(&xv);
        uint32_t* ou = reinterpret_cast<uint32_t*>(&out[q]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 xf = unpack_bf16x2(xu[e]);
          const int k0 = q * 8 + 2 * e;
          const float y0 = __uint_as_float(yd[k0]) + ef * __uint_as_float(yf[k0]) + eb * __uint_as_float(yb[k0]) + D2 * xf.x;
          const float y1 = __uint_as_float(yd[k0 + 1]) + ef * __uint_as_float(yf[k0 + 1]) +
                           eb * __uint_as_float(yb[k0 + 1]) + D2 * xf.y;
          ou[e] = pack_bf16x2(y0, y1);
        }
      }
      uint4* dst = reinterpret_cast<uint4*>(yrow + pc * 32);
#pragma unroll
      for (int q = 0; q < 4; ++q) dst[q] = out[q];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mate
