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
//
// fp16 x.  When the x rows are fp16 (the block stores its projected x in fp16), the output kernel forms M
// with packed fp16 multiplies from fp16 column-factor tables and runs M x as an fp16 MMA: fewer ALU
// operations per element and an intra-chunk operand 8 times finer than bf16.  |M_ij| = |C_i . B_j| delta_j
// dec(i, j) must then stay below 65504 (the products are not saturated).  With bf16 x (the standalone entry
// points) M is formed in fp32 and rounded once to bf16.
//
// Precision.  States, decays and accumulations are fp32.  The chunk states S are stored in fp32; the
// carried states H, an operand of the C H^T product, are stored as a bf16 pair hi + lo (hi = bf16(H),
// lo = bf16(H - hi)) and multiplied as two accumulating products, which keeps about 16 bits of H.  G and
// the state products' operands (the decay-weighted x and B) are fp16 (11 bits), so M = G delta dec is
// rounded once, to the bf16 MMA operand, from an fp16 G that is already 8 times finer than bf16.  fp16
// conversions saturate at +-65504 (|C_i . B_j| and |delta_j x_j| stay far below that for these blocks).
// Rows are gathered through the scan-order map (the permutation is done by addressing) and y is
// stored back at grid-order rows.
#pragma once
#include "common.cuh"
#include "simt.cuh"

namespace mate {

constexpr int kSsdQ = 256;   // chunk length of the tensor-core scan
constexpr int kSsdP = 64;    // head size
constexpr int kSsdN = 128;   // state size

// Decay tables of one (video chunk, head, 128-row tile t), written by the state kernel and read by the
// output kernel, in floats.  Row fields are indexed by the tile row r (token i = 128 t + r), column
// fields by the chunk column j:
//   uf, ub   row factors exp(s_i - s_{64 ib - 1}), exp(s'_{64 ib + 64} - s'_i) of row block ib = i / 64
//   si, sx   s_i log2(e), s'_i log2(e)               ef, eb  exp(s_i), exp(s_last - s'_i)
//   dl       delta_i                                  wf, wb  [2][256] column factors of row blocks 2t, 2t + 1
//                                                             (fp16, first half of the slot, for fp16 x)
//   lf, lb   log2(delta_j) - s_j log2(e), log2(delta_j) + s'_j log2(e) for the tile's own columns
// (s inclusive and s' = s - delta A exclusive cumulative sums of delta A over the chunk).
constexpr int kTUf = 0, kTUb = 128, kTSi = 256, kTSx = 384, kTEf = 512, kTEb = 640, kTDl = 768, kTWf = 896,
              kTWb = 1408, kTLf = 1920, kTLb = 2048, kOutTbl = 2176;
constexpr float kLog2e = 1.4426950408889634f;

struct SsdBf16Params {
  SeqRows s;
  int B, nh, nRc, nVc;
  const float* A_log;
  const float* Dp;
  __half* Gm;         // [B][nVc][Q][Q]  C B^T of each video chunk in fp16 (off-diagonal use)
  float* Gd;          // [B][nVc][Q]     its diagonal C_i . B_i in fp32
  float* Sf;          // [B][nRc + nVc][nh][N][P]   (states are stored transposed: n-major, p fastest)
  float* Sb;          // [B][nVc][nh][N][P]
  float* gl;          // [B][nRc + nVc][nh]  s_last of each chunk
  __nv_bfloat16* Hf;  // [B][nVc][nh][2][N][P]  state entering video chunk v, forward traversal, as hi | lo
  __nv_bfloat16* Hb;  // [B][nVc][nh][2][N][P]  state entering video chunk v, backward traversal, as hi | lo
  int* crow;          // [B][nVc][Q]     source row of each video-chunk row (-1 past the end)
  float* tbl;         // [B][nVc][nh][2][kOutTbl]  decay tables of each 128-row tile (layout below)
  // Optional separate parameters of the backward scan (null: shared with the forward scan).  With them,
  // the backward delta sits at column s.db_off of the delta rows, glb holds the backward log-decays and
  // Srb the review chunks' states under the backward parameters (the backward scan also runs over the
  // review prefix first, in its stored order).
  const float* A_log_b;
  const float* Dp_b;
  float* glb;           // [B][nRc + nVc][nh]
  float* Srb;           // [B][nRc][nh][N][P]
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
  // a wait that ran out (flagged in the status word) skips the read-out; the CTA still frees its TMEM
  const bool ok = !__syncthreads_or(!mbar_wait(bar, 0));
  tc_fence_after();
  const int i = t * 128 + warp * 32 + lane;
  __half* grow = p.Gm + ((static_cast<long long>(b) * p.nVc + v) * kSsdQ + i) * kSsdQ;
  for (int c0 = 0; c0 < 256 && ok; c0 += 32) {
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
      pk.x = pack_f16x2_sat(__uint_as_float(r[q * 8 + 0]), __uint_as_float(r[q * 8 + 1]));
      pk.y = pack_f16x2_sat(__uint_as_float(r[q * 8 + 2]), __uint_as_float(r[q * 8 + 3]));
      pk.z = pack_f16x2_sat(__uint_as_float(r[q * 8 + 4]), __uint_as_float(r[q * 8 + 5]));
      pk.w = pack_f16x2_sat(__uint_as_float(r[q * 8 + 6]), __uint_as_float(r[q * 8 + 7]));
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
// Chunk-local end states, persistent and pipelined.  grid = min(B (nRc + nVc), SMs), kStThreads threads;
// each CTA walks the chunks w = blockIdx.x, blockIdx.x + gridDim.x, ... (w = b (nRc + nVc) + c) and,
// inside a chunk, every head.  The roles overlap one head's x loads, MMAs and state stores with the next
// head's scan and weighting:
//   warps 0..3   drain: a head's two states from TMEM (lane quadrant = warp, lane = state row n) through
//                a 4 KB transpose buffer per warp (32 rows x 32 columns at a time) to the fp32 state arrays
//                as whole 128-byte row segments, then release the accumulator set
//   warps 4..11  prep (thread j = token j of the chunk): per chunk the B rows (bf16 -> fp16, into the
//                tile read MN-major as the A operand); per head the decay scan, the output kernel's decay
//                tables and the decay-weighted x tiles (fp16, MN-major) from the head's x tile
//   warp 12      MMA issue (lane 0): D[n][p] = sum_j B[j][n] (w_j x[j][p]), M = N_state = 128, N = P = 64,
//                K = Q = 256, for both directions into one of two TMEM accumulator sets [Sf | Sb]
//   warp 13      x loader: each head's 256 x rows (64 columns, TMA four-row gathers through the scan-order
//                row map) into a ring of two tiles, two heads ahead of the weighting
// ---------------------------------------------------------------------------------------------------
constexpr int kStPrepWarp0 = 4, kStMmaWarp = 12, kStLoadWarp = 13, kStThreads = 448;
constexpr uint32_t kStOffX = 65536;                 // weighted x: fwd 32 KB | bwd 32 KB
constexpr uint32_t kStOffXr = kStOffX + 65536;      // x tiles as loaded, two of 32 KB
constexpr uint32_t kStOffW = kStOffXr + 65536;      // weights of the current head: fwd [256], bwd [256]
constexpr uint32_t kStOffRow = kStOffW + 2048;      // source rows of the chunk [256]
constexpr uint32_t kStOffMisc = kStOffRow + 2048;   // scan warp totals [8], row-block boundaries [8]
constexpr uint32_t kStOffStage = kStOffMisc + 64;   // drain transpose buffers, 4 KB per drain warp
constexpr uint32_t kStOffBar = kStOffStage + 4 * 4096;
constexpr uint32_t kStSmem = kStOffBar + 128;
static_assert(kStSmem + 1024 <= 232448, "shared memory of the state kernel");

// Inclusive prefix sum of one value per prep thread (j = 0..255) on named barrier `id`.
__device__ __forceinline__ float prep_scan_256(float v, float* warp_tot, int j, int id) {
  const int lane = j & 31, w = j >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float u = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += u;
  }
  if (lane == 31) warp_tot[w] = v;
  named_bar_sync(id, 256);
  float base = 0.f;
  for (int k = 0; k < w; ++k) base += warp_tot[k];
  named_bar_sync(id, 256);
  return v + base;
}

// x rows of the state kernel: review and video arrays (one-row boxes of 64 columns, for four-row gathers).
struct SsdStateMaps {
  CUtensorMap xv, xr;
  int rows_v, rows_r;   // row extents; gathers of rows past a partial chunk's end use them (zeros)
};

template <bool XF16>
__global__ void __launch_bounds__(kStThreads, 1) ssd_state_kernel(const SsdBf16Params p,
                                                                  const __grid_constant__ SsdStateMaps mp) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem;   // [256 j][128 n] fp16
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStOffBar);
  uint64_t* x_full = bars;          // weighted x (and, for a chunk's first head, the B tile): 256 prep threads
  uint64_t* x_empty = bars + 1;     // MMA commit
  uint64_t* acc_full = bars + 2;    // [2] MMA commit -> drain
  uint64_t* acc_empty = bars + 4;   // [2] 4 drain warps -> MMA
  uint64_t* xr_full = bars + 6;     // [2] x tile bytes
  uint64_t* xr_empty = bars + 8;    // [2] 256 prep threads have read the tile
  uint32_t* slot = reinterpret_cast<uint32_t*>(bars + 10);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nC = p.nRc + p.nVc, nwork = p.B * nC, nh = p.nh;
  const bool per_dir = p.A_log_b != nullptr;   // backward scan with its own A, D and delta

  if (threadIdx.x == 0) {
    mbar_init(x_full, 256);
    mbar_init(x_empty, 1);
    for (int q = 0; q < 2; ++q) {
      mbar_init(&acc_full[q], 1);
      mbar_init(&acc_empty[q], 4);
      mbar_init(&xr_full[q], 1);
      mbar_init(&xr_empty[q], 256);
    }
    mbar_fence_init();
  }
  if (warp == kStMmaWarp) tmem_alloc(slot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;

  if (warp < kStPrepWarp0) {
    // ------------------------------------------------------------------------------ drain
    float4* stage = reinterpret_cast<float4*>(smem + kStOffStage + warp * 4096);
    int u = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
      const int c = w % nC, b = w / nC;
      const bool video = c >= p.nRc;
      for (int h = 0; h < nh; ++h, ++u) {
        const int acc = u & 1, use = u >> 1;
        if (!mbar_wait(&acc_full[acc], use & 1)) { ok = false; break; }
        tc_fence_after();
        for (int dir = 0; dir < 2; ++dir) {
          if (dir == 1 && !video && !per_dir) break;
          float* dst = dir == 0
              ? p.Sf + ((static_cast<long long>(b) * nC + c) * nh + h) * (kSsdP * kSsdN)
              : (video ? p.Sb + ((static_cast<long long>(b) * p.nVc + (c - p.nRc)) * nh + h) * (kSsdP * kSsdN)
                       : p.Srb + ((static_cast<long long>(b) * p.nRc + c) * nh + h) * (kSsdP * kSsdN));
          // lane = state row n holds 32 p values per load; the warp's 32 rows x 32 columns go through its
          // transpose buffer (16-byte chunk c of row r at chunk c ^ (r & 7): conflict-free both ways) so
          // that each store instruction writes four whole 128-byte row segments of the [N][P] state
          for (int pc = 0; pc < 2; ++pc) {
            uint32_t r[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + acc * 128 + dir * 64 + pc * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 8; ++q)
              stage[lane * 8 + (q ^ (lane & 7))] =
                  make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                              __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int row = k * 4 + (lane >> 3), q = lane & 7;
              reinterpret_cast<float4*>(dst + (warp * 32 + row) * kSsdP + pc * 32)[q] = stage[row * 8 + (q ^ (row & 7))];
            }
            __syncwarp();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
      }
    }
  } else if (warp < kStMmaWarp) {
    // ------------------------------------------------------------------------------ prep
    const int j = threadIdx.x - kStPrepWarp0 * 32;
    float* sWf = reinterpret_cast<float*>(smem + kStOffW);
    float* sWb = sWf + 256;
    long long* srow = reinterpret_cast<long long*>(smem + kStOffRow);
    float* wtot = reinterpret_cast<float*>(smem + kStOffMisc);
    float* bnd = wtot + 8;   // s at the ends of row blocks 0..2, s' at the starts of 1..3
    int u = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
      const int c = w % nC, b = w / nC;
      const ChunkBase cb = chunk_base(p.s, c, p.nRc);
      const bool video = c >= p.nRc;
      named_bar_sync(1, 256);   // every prep thread is done with the previous chunk's rows
      {
        const RowRef rr = chunk_row(p.s, b, c, p.nRc, j);
        srow[j] = rr.valid ? rr.r : -1;
      }
      named_bar_sync(1, 256);
      const long long myrw = srow[j];
      uint4 bv[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int it = j + e * 256;
        const long long rw = srow[it >> 4];
        bv[e] = rw >= 0 ? __ldg(reinterpret_cast<const uint4*>(cb.b + rw * cb.ldb) + (it & 15)) : make_uint4(0, 0, 0, 0);
      }
      // the previous chunk's MMAs (all committed before its last head's x_empty) must be done with the B tile
      if (u > 0) ok = mbar_wait(x_empty, (u - 1) & 1);
      if (named_bar_any(1, 256, !ok)) { ok = false; break; }
#pragma unroll
      for (int e = 0; e < 16; ++e) {   // bf16 -> fp16 (zeros past a partial chunk's end)
        const int it = j + e * 256;
        const uint32_t* bw = reinterpret_cast<const uint32_t*>(&bv[e]);
        uint4 o;
        uint32_t* po = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = unpack_bf16x2(bw[k]);
          po[k] = pack_f16x2_sat(f.x, f.y);
        }
        *reinterpret_cast<uint4*>(sB + sw128_kmajor_offset(it >> 4, (it & 15) * 8, 32768)) = o;
      }
      float dl_next = myrw >= 0 ? cb.d[myrw * cb.ldd] : 0.f;
      float dlb_next = per_dir ? (myrw >= 0 ? cb.d[myrw * cb.ldd + p.s.db_off] : 0.f) : dl_next;
      float alog_next = p.A_log[0];
      for (int h = 0; h < nh; ++h, ++u) {
        const float A = -__expf(alog_next);
        const float dl = dl_next, dlb = dlb_next;
        if (h + 1 < nh) {   // the next head's deltas and A: a whole head of work to arrive
          dl_next = myrw >= 0 ? cb.d[myrw * cb.ldd + h + 1] : 0.f;
          dlb_next = per_dir ? (myrw >= 0 ? cb.d[myrw * cb.ldd + p.s.db_off + h + 1] : 0.f) : dl_next;
          alog_next = p.A_log[h + 1];
        }
        const float a = dl * A;
        const float s = prep_scan_256(a, wtot, j, 1);
        if (j == 255) wtot[8 - 1] = s;   // slot 7 holds s_last once the scan is done with the warp totals
        if ((j & 63) == 63 && j < 255) bnd[j >> 6] = s;   // bnd[ib - 1] = s_{64 ib - 1}, ib = 1..3
        named_bar_sync(1, 256);
        const float s_last = wtot[7];
        // backward scan quantities: the same as the forward ones unless the backward parameters differ
        float ab = a, sbk = s, sb_last = s_last;
        if (per_dir) {
          ab = dlb * -__expf(p.A_log_b[h]);
          named_bar_sync(1, 256);   // every thread has read s_last before the second scan reuses wtot
          sbk = prep_scan_256(ab, wtot, j, 1);
          if (j == 255) wtot[8 - 1] = sbk;
          named_bar_sync(1, 256);
          sb_last = wtot[7];
        }
        const float sx = sbk - ab;   // exclusive backward cumulative sum s'
        if ((j & 63) == 0 && j > 0) bnd[4 + (j >> 6) - 1] = sx;   // bnd[4 + ib] = s'_{64 ib + 64}, ib = 0..2
        named_bar_sync(1, 256);
        if (video) {
          // decay tables of the output kernel (see kOutTbl)
          const long long cv = static_cast<long long>(b) * p.nVc + (c - p.nRc);
          if (h == 0) p.crow[cv * kSsdQ + j] = myrw >= 0 ? static_cast<int>(myrw) : -1;
          float* T0 = p.tbl + (cv * nh + h) * 2 * kOutTbl;
          float* T = T0 + (j >> 7) * kOutTbl;
          const int r = j & 127, ib = j >> 6;
          T[kTUf + r] = ib > 0 ? __expf(s - bnd[ib - 1]) : 0.f;
          T[kTUb + r] = ib < 3 ? __expf(bnd[4 + ib] - sx) : 0.f;
          T[kTSi + r] = s * kLog2e;
          T[kTSx + r] = sx * kLog2e;
          T[kTEf + r] = __expf(s);
          T[kTEb + r] = __expf(sb_last - sx);
          T[kTDl + r] = 0.5f * (dl + dlb);   // the output epilogue's diagonal term uses 2 (D + G_ii dl)
          const float l2d = dl > 0.f ? __log2f(dl) : -INFINITY;
          const float l2db = dlb > 0.f ? __log2f(dlb) : -INFINITY;
          T[kTLf + r] = l2d - s * kLog2e;
          T[kTLb + r] = l2db + sx * kLog2e;
#pragma unroll
          for (int q = 0; q < 4; ++q) {   // column factors of row block q (stored with the tile holding it)
            const float wfv = (q > 0 && j < 64 * q) ? dl * __expf(bnd[q - 1] - s) : 0.f;
            const float wbv = (q < 3 && j >= 64 * q + 64) ? dlb * __expf(sx - bnd[4 + q]) : 0.f;
            if (XF16) {
              float* Tq = T0 + (q >> 1) * kOutTbl;
              reinterpret_cast<__half*>(Tq + kTWf)[(q & 1) * 256 + j] = __float2half_rn(wfv);
              reinterpret_cast<__half*>(Tq + kTWb)[(q & 1) * 256 + j] = __float2half_rn(wbv);
            } else {
              float* W = T0 + (q >> 1) * kOutTbl + (q & 1) * 256 + j;
              W[kTWf] = wfv;
              W[kTWb] = wbv;
            }
          }
        }
        if (j == 0) {
          p.gl[(static_cast<long long>(b) * nC + c) * nh + h] = s_last;
          if (per_dir) p.glb[(static_cast<long long>(b) * nC + c) * nh + h] = sb_last;
        }
        sWf[j] = __expf(s_last - s) * dl;
        // second product: the backward state of a video chunk (decay to its start); for a review chunk
        // under separate backward parameters, its state at the chunk end under those parameters
        sWb[j] = (video || !per_dir) ? __expf(sx) * dlb : __expf(sb_last - sbk) * dlb;
        const int xb = u & 1;
        // the previous head's MMAs are done with the weighted tiles, and this head's x tile has landed
        ok = mbar_wait(x_empty, (u & 1) ^ 1) && mbar_wait(&xr_full[xb], (u >> 1) & 1);
        if (named_bar_any(1, 256, !ok)) { ok = false; break; }
        uint8_t* sXf = smem + kStOffX;
        uint8_t* sXb = sXf + 32768;
        const uint8_t* sXr = smem + kStOffXr + xb * 32768;
#pragma unroll
        for (int e = 0; e < 8; ++e) {   // weighted x tiles, 8 values (one 16-byte chunk) per item
          const int it = j + e * 256;
          const int r = it >> 3, ch = it & 7;
          const float wf = sWf[r], wb = sWb[r];
          const uint32_t off = sw128_mnmajor_offset(r, ch * 8, 32768);
          const uint4 xv = *reinterpret_cast<const uint4*>(sXr + off);
          const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xv);
          uint4 of, ob;
          uint32_t* pf = reinterpret_cast<uint32_t*>(&of);
          uint32_t* pb = reinterpret_cast<uint32_t*>(&ob);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = XF16 ? unpack_f16x2(xw[k]) : unpack_bf16x2(xw[k]);
            pf[k] = pack_f16x2_sat(f.x * wf, f.y * wf);
            pb[k] = pack_f16x2_sat(f.x * wb, f.y * wb);
          }
          *reinterpret_cast<uint4*>(sXf + off) = of;
          *reinterpret_cast<uint4*>(sXb + off) = ob;
        }
        fence_proxy_async();
        mbar_arrive(x_full);
        mbar_arrive(&xr_empty[xb]);
      }
    }
  } else if (warp == kStMmaWarp) {
    // ------------------------------------------------------------------------------ MMA issue
    if (lane == 0) {
      // both directions as one N = 128 product: B = [Xf | Xb], two MN blocks 32 KB apart -> [Sf | Sb];
      // N = 64 (Xf only) for a review chunk without a backward state
      const uint32_t idesc2 = idesc_f16_f32(128, 128, 1, 1), idesc1 = idesc_f16_f32(128, 64, 1, 1);
      const uint32_t ab = smem_u32(sB);
      int u = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
        const bool two = (w % nC) >= p.nRc || per_dir;   // a backward state for this chunk
        for (int h = 0; h < nh; ++h, ++u) {
          const int buf = u & 1, use = u >> 1;
          if (!mbar_wait(x_full, u & 1) || !mbar_wait(&acc_empty[buf], (use & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t xf = smem_u32(smem + kStOffX);
          const uint32_t d = tmem + buf * 128;
#pragma unroll 4
          for (int k = 0; k < 16; ++k)
            mma_bf16_ss(d, desc_sw128(ab + k * 2048, 32768, 1024), desc_sw128(xf + k * 2048, 32768, 1024),
                        two ? idesc2 : idesc1, k > 0);
          mma_commit(x_empty);
          mma_commit(&acc_full[buf]);
        }
      }
    }
    __syncwarp();
  } else if (warp == kStLoadWarp) {
    // ------------------------------------------------------------------------------ x loader
    // every exit decision is warp-uniform (a lane leaving alone would strand __syncwarp)
    auto wait_all = [&](uint64_t* bar, unsigned parity) { return !__any_sync(0xffffffffu, !mbar_wait(bar, parity)); };
    int u = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < nwork && ok; w += gridDim.x) {
      const int c = w % nC, b = w / nC;
      const bool video = c >= p.nRc;
      const CUtensorMap* map = video ? &mp.xv : &mp.xr;
      int id[8];   // chunk rows 8 lane .. 8 lane + 7 (rows past a partial chunk's end: the map's extent)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const RowRef rr = chunk_row(p.s, b, c, p.nRc, 8 * lane + e);
        id[e] = rr.valid ? static_cast<int>(rr.r) : (video ? mp.rows_v : mp.rows_r);
      }
      for (int h = 0; h < nh; ++h, ++u) {
        const int xb = u & 1, use = u >> 1;
        if (!wait_all(&xr_empty[xb], (use & 1) ^ 1)) { ok = false; break; }
        if (lane == 0) mbar_arrive_expect_tx(&xr_full[xb], 32768);
        __syncwarp();
        uint8_t* dst = smem + kStOffXr + xb * 32768;
        tma_gather4(map, &xr_full[xb], dst + (2 * lane) * 512, h * kSsdP, id[0], id[1], id[2], id[3]);
        tma_gather4(map, &xr_full[xb], dst + (2 * lane + 1) * 512, h * kSsdP, id[4], id[5], id[6], id[7]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kStMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------------------------------
// Sequential carry across chunks.  grid (P*N/8/128, nh, 2*B), 128 threads; thread = 8 state elements.
// Review chunks are visited first (same order in both directions); then the video chunks ascending
// (forward) or descending (backward).  Reads the fp32 chunk states and writes the state entering each
// video chunk as the bf16 pair hi | lo (hi = bf16(H), lo = bf16(H - hi)).
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
  auto step = [&](float glv, float4 s0, float4 s1) {
    const float g = __expf(glv);
    H[0] = fmaf(g, H[0], s0.x); H[1] = fmaf(g, H[1], s0.y); H[2] = fmaf(g, H[2], s0.z); H[3] = fmaf(g, H[3], s0.w);
    H[4] = fmaf(g, H[4], s1.x); H[5] = fmaf(g, H[5], s1.y); H[6] = fmaf(g, H[6], s1.z); H[7] = fmaf(g, H[7], s1.w);
  };
  auto store = [&](__nv_bfloat16* base) {   // base: the [2][N][P] hi | lo pair of one (chunk, head)
    uint4 hi, lo;
    uint32_t* uh = reinterpret_cast<uint32_t*>(&hi);
    uint32_t* ul = reinterpret_cast<uint32_t*>(&lo);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uh[e] = pack_bf16x2(H[2 * e], H[2 * e + 1]);
      const float2 r = unpack_bf16x2(uh[e]);
      ul[e] = pack_bf16x2(H[2 * e] - r.x, H[2 * e + 1] - r.y);
    }
    *reinterpret_cast<uint4*>(base + e8 * 8) = hi;
    *reinterpret_cast<uint4*>(base + PN + e8 * 8) = lo;
  };
  auto load = [&](const float* S, float4& s0, float4& s1) {
    s0 = __ldg(reinterpret_cast<const float4*>(S) + 2 * e8);
    s1 = __ldg(reinterpret_cast<const float4*>(S) + 2 * e8 + 1);
  };
  const bool bwd_own = dir == 1 && p.A_log_b != nullptr;   // backward scan with its own parameters
  const float* gld = bwd_own ? p.glb : p.gl;
  for (int c = 0; c < p.nRc; ++c) {
    const long long ci = (static_cast<long long>(b) * nC + c) * p.nh + h;
    const float* S = bwd_own ? p.Srb + ((static_cast<long long>(b) * p.nRc + c) * p.nh + h) * PN : p.Sf + ci * PN;
    float4 s0, s1;
    load(S, s0, s1);
    step(gld[ci], s0, s1);
  }
  constexpr int U = 8;   // chunks in flight per thread (256 bytes of fp32 state)
  for (int k0 = 0; k0 < p.nVc; k0 += U) {
    float4 sv[U][2];
    float gv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + u;
      if (k < p.nVc) {
        const int v = dir == 0 ? k : p.nVc - 1 - k;
        const long long ci = (static_cast<long long>(b) * nC + p.nRc + v) * p.nh + h;
        const long long vi = (static_cast<long long>(b) * p.nVc + v) * p.nh + h;
        gv[u] = gld[ci];
        load(dir == 0 ? p.Sf + ci * PN : p.Sb + vi * PN, sv[u][0], sv[u][1]);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + u;
      if (k < p.nVc) {
        const int v = dir == 0 ? k : p.nVc - 1 - k;
        const long long vi = (static_cast<long long>(b) * p.nVc + v) * p.nh + h;
        store((dir == 0 ? p.Hf : p.Hb) + vi * 2 * PN);
        step(gv[u], sv[u][0], sv[u][1]);
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------------
// Outputs of the video chunks: persistent, warp-specialised.  A group = (sample, video chunk, 128-row
// tile t); a CTA walks groups blockIdx.x, blockIdx.x + gridDim.x, ... and within a group all heads in
// turn (one work item per head).  The tile's rows of G = C B^T and of C are the same for every head, so
// they are loaded once per group and stay in shared memory.
//
//   warp 0       per item: the head's decay tables (one bulk copy) and x rows (all 256 of the chunk,
//                MN-major, TMA four-row gathers) into one of two x buffers.
//   warp 1       per group: the tile's C rows (K-major, four-row gathers); per item: the head's incoming
//                states as four [N = 128][P = 64] blocks, Hf hi, Hb hi, Hf lo, Hb lo (MN-major, 2D TMA),
//                through a ring of three 16 KB slots, so that up to three are in flight.
//   warp 2       per group: the tile's rows of G (2D TMA) into four 64-column slots, each refilled once
//                the last head of the previous group has read it.
//   warp 3       MMA issue (lane 0 only; an issuing thread stalls while the tensor pipe is busy, so it has
//                no other work): Yd = M x per K half of M (A from TMEM) and, after each half, two of the
//                four N = 64 products Yf (+)= C Hf^T, Yb (+)= C Hb^T (hi parts, then lo parts), into one of
//                two TMEM accumulator sets.
//   warps 4..11  transform (two warps per TMEM lane quadrant, each taking 16 contiguous TMEM columns of
//                every 64-element column block, stored with one TMEM store): form
//                M_ij = G_ij delta_j dec(i, j) (diagonal excluded) from the G slots and store M straight
//                into TMEM as the A operand of the MMA (two bf16 per 32-bit column), in two K halves.
//   warps 12..15 epilogue: y_i = Yd + exp(s_i) Yf + exp(s_last - s'_i) Yb + 2 (D + G_ii delta_i) x_i,
//                stored at the grid-order row of the token.
//
// Decay factors: for a 64-row block ib and a column j of an EARLIER 64-block (forward direction), the
// reference k = 64 ib - 1 lies between them, so exp(s_i - s_j) = exp(s_i - s_k) exp(s_k - s_j) (both
// exponents <= 0): a per-row factor times a per-(ib, j) column factor.  Columns of LATER blocks use
// k' = 64 (ib + 1) with the exclusive sums.  Only the 64 x 64 diagonal blocks need one exponential per
// element, taken in the log2 domain: delta_j exp(s_i - s_j) = 2^(s_i log2e + lf_j) below the diagonal,
// delta_j exp(s'_j - s'_i) = 2^(lb_j - s'_i log2e) above it.
// TMEM columns: [0, 128) M; accumulator set a at 128 + 192 a: Yd [+0, +64), Yf [+64, +128), Yb [+128, +192).
// ---------------------------------------------------------------------------------------------------
constexpr int kOutLoadWarps = 3, kOutXformWarps = 8, kOutEpiWarps = 4;
constexpr int kOutMmaWarp = kOutLoadWarps;                                    // issues from its lane 0
constexpr int kOutFirstXformWarp = kOutMmaWarp + 1, kOutFirstEpiWarp = kOutFirstXformWarp + kOutXformWarps;
constexpr int kSsdOutThreads = (kOutFirstEpiWarp + kOutEpiWarps) * 32;        // 512
static_assert(kOutFirstXformWarp % 4 == 0 && kOutFirstEpiWarp % 4 == 0, "TMEM lane quadrants follow warp % 4");

// shared memory map (offsets from the 1024-aligned base)
constexpr uint32_t kOutTblBytes = kOutTbl * 4;         // 8704
constexpr uint32_t kOutXBuf = 32768;                    // x tile of one item, two of them
constexpr uint32_t kOutOffTbl = 2 * kOutXBuf;           // the item's decay tables, two of them
constexpr uint32_t kOutOffC = kOutOffTbl + 2 * kOutTblBytes;   // C rows of the tile: 2 K blocks of 16 KB
constexpr uint32_t kOutHSlots = 3;                      // ring of [N = 128][P = 64] state blocks
constexpr uint32_t kOutOffH = kOutOffC + 32768;
constexpr uint32_t kOutOffG = kOutOffH + kOutHSlots * 16384;   // 4 slots of [128 rows][64 cols] K-major
constexpr uint32_t kOutOffBar = kOutOffG + 4 * 16384;
constexpr uint32_t kOutSmem = kOutOffBar + 256;
static_assert(kOutOffC % 1024 == 0 && kOutOffH % 1024 == 0 && kOutOffG % 1024 == 0, "1024-byte operand tiles");
static_assert(kOutSmem + 1024 <= 232448, "shared memory of the output kernel");

// Tensor maps of the output kernel: x and C rows of the video arrays (one-row boxes of 64 columns, for
// four-row gathers), the carried states ([2][N rows][P] hi | lo per chunk and head, 64 x 128 boxes) and G
// ([chunk rows][Q] fp16, 64 x 128 boxes).
struct SsdOutMaps {
  CUtensorMap x, c, hf, hb, g;
  int rows;   // row extent of the x / C maps; gathers of invalid rows use this (out of range -> zeros)
};

template <bool XF16>
__global__ void __launch_bounds__(kSsdOutThreads, 1) ssd_output_kernel(const SsdBf16Params p,
                                                                        const __grid_constant__ SsdOutMaps mp) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOutOffBar);
  uint64_t* x_full = bars;         // [2] x + table bytes
  uint64_t* x_empty = bars + 2;    // [2] last Yd MMA commit (the epilogue reads its x rows and table
                                   //     entries from global memory, so the buffer never waits for it)
  uint64_t* h_full = bars + 4;     // [3] one state block's bytes
  uint64_t* h_empty = bars + 7;    // [3] the Yf / Yb MMA commit that read the slot
  uint64_t* c_full = bars + 10;    // C bytes (per group)
  uint64_t* c_empty = bars + 11;   // last head's Yf / Yb MMA commit
  uint64_t* g_full = bars + 12;    // [4] one G slot's bytes (per group)
  uint64_t* g_empty = bars + 16;   // [4] the 8 transform warps have read the slot for the last head
  uint64_t* m_full = bars + 20;    // [2] per K half of M: transform -> MMA (count 256)
  uint64_t* m_empty = bars + 22;   // [2] per K half of M: MMA commit -> transform
  uint64_t* y_full = bars + 24;    // [2] MMA commit -> epilogue
  uint64_t* y_empty = bars + 26;   // [2] epilogue warps -> MMA (count 4)
  uint32_t* slot = reinterpret_cast<uint32_t*>(bars + 28);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nh = p.nh;
  const int ngroups = p.B * p.nVc * 2;

  if (threadIdx.x == 0) {
    for (int q = 0; q < 2; ++q) {
      mbar_init(&x_full[q], 1);
      mbar_init(&x_empty[q], 1);
      mbar_init(&m_full[q], kOutXformWarps * 32);
      mbar_init(&m_empty[q], 1);
      mbar_init(&y_full[q], 1);
      mbar_init(&y_empty[q], kOutEpiWarps);
    }
    for (int q = 0; q < 3; ++q) {
      mbar_init(&h_full[q], 1);
      mbar_init(&h_empty[q], 1);
    }
    mbar_init(c_full, 1);
    mbar_init(c_empty, 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&g_full[q], 1);
      mbar_init(&g_empty[q], kOutXformWarps);
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

  auto decode = [&](int g, int& b, int& v, int& t) {
    t = g & 1;
    const int rest = g >> 1;
    v = rest % p.nVc;
    b = rest / p.nVc;
  };
  // every exit decision inside a warp is warp-uniform (a lane leaving alone would strand __syncwarp)
  auto wait_all = [&](uint64_t* bar, unsigned parity) { return !__any_sync(0xffffffffu, !mbar_wait(bar, parity)); };

  if (warp == 0) {
    // ------------------------------------------------------------------------------ x, tables, H
    int rows[8], rows_next[8];   // chunk rows 8 lane .. 8 lane + 7 of the current / next group
    auto fetch_rows = [&](int g, int (&rw)[8]) {
      if (g >= ngroups) return;
      int b, v, t;
      decode(g, b, v, t);
      const int4* src = reinterpret_cast<const int4*>(p.crow + (static_cast<long long>(b) * p.nVc + v) * kSsdQ);
      const int4 a0 = src[2 * lane], a1 = src[2 * lane + 1];
      rw[0] = a0.x; rw[1] = a0.y; rw[2] = a0.z; rw[3] = a0.w;
      rw[4] = a1.x; rw[5] = a1.y; rw[6] = a1.z; rw[7] = a1.w;
    };
    fetch_rows(blockIdx.x, rows);
    int k = 0;
    bool ok = true;
    for (int g = blockIdx.x; g < ngroups && ok; g += gridDim.x) {
      int b, v, t;
      decode(g, b, v, t);
      const long long cidx = static_cast<long long>(b) * p.nVc + v;
      fetch_rows(g + gridDim.x, rows_next);
      for (int h = 0; h < nh; ++h, ++k) {
        const int buf = k & 1, use = k >> 1;
        if (!wait_all(&x_empty[buf], (use & 1) ^ 1)) { ok = false; break; }
        uint8_t* XB = smem + buf * kOutXBuf;
        if (lane == 0) {
          mbar_arrive_expect_tx(&x_full[buf], 32768 + kOutTblBytes);
          bulk_load(smem + kOutOffTbl + buf * kOutTblBytes, p.tbl + ((cidx * nh + h) * 2 + t) * kOutTbl, kOutTblBytes,
                    &x_full[buf]);
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 2; ++u) {   // 4 rows per gather, 8 rows per lane
          int id[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) id[e] = rows[4 * u + e] < 0 ? mp.rows : rows[4 * u + e];
          tma_gather4(&mp.x, &x_full[buf], XB + (2 * lane + u) * 512, h * kSsdP, id[0], id[1], id[2], id[3]);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) rows[e] = rows_next[e];
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------------------ C rows per group, H per item
    int kg = 0, k = 0;
    bool ok = true;
    for (int g = blockIdx.x; g < ngroups && ok; g += gridDim.x, ++kg) {
      int b, v, t;
      decode(g, b, v, t);
      const long long cidx = static_cast<long long>(b) * p.nVc + v;
      const int4 r4 = reinterpret_cast<const int4*>(p.crow + cidx * kSsdQ + t * 128)[lane];
      const int id[4] = {r4.x < 0 ? mp.rows : r4.x, r4.y < 0 ? mp.rows : r4.y, r4.z < 0 ? mp.rows : r4.z,
                         r4.w < 0 ? mp.rows : r4.w};
      if (!wait_all(c_empty, (kg & 1) ^ 1)) break;
      if (lane == 0) mbar_arrive_expect_tx(c_full, 32768);
      __syncwarp();
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
        tma_gather4(&mp.c, c_full, smem + kOutOffC + kb * 16384 + lane * 512, kb * 64, id[0], id[1], id[2], id[3]);
      for (int h = 0; h < nh && ok; ++h, ++k) {
        for (int q = 0; q < 4; ++q) {   // Hf hi, Hb hi, Hf lo, Hb lo through the ring of three slots
          const int u = 4 * k + q, sl = u % 3, use = u / 3;
          if (!wait_all(&h_empty[sl], (use & 1) ^ 1)) { ok = false; break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(&h_full[sl], 16384);
            const int hrow = static_cast<int>(((cidx * nh + h) * 2 + (q >> 1)) * kSsdN);
            tma_load_2d((q & 1) ? &mp.hb : &mp.hf, &h_full[sl], smem + kOutOffH + sl * 16384, 0, hrow);
          }
          __syncwarp();
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------------------------ G rows, per group
    if (lane == 0) {
      int kg = 0;
      bool ok = true;
      for (int g = blockIdx.x; g < ngroups && ok; g += gridDim.x, ++kg) {
        int b, v, t;
        decode(g, b, v, t);
        const int grow = static_cast<int>((static_cast<long long>(b) * p.nVc + v) * kSsdQ + t * 128);
        for (int cb = 0; cb < 4 && ok; ++cb) {
          ok = mbar_wait(&g_empty[cb], (kg & 1) ^ 1);
          if (ok) {
            mbar_arrive_expect_tx(&g_full[cb], 16384);
            tma_load_2d(&mp.g, &g_full[cb], smem + kOutOffG + cb * 16384, cb * 64, grow);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == kOutMmaWarp) {
    // ------------------------------------------------------------------------------ MMA issue
    if (lane == 0) {
      // Yd: N = P, fp16 operands when x is fp16
      const uint32_t idesc_d = XF16 ? idesc_f16_f32(128, 64, 0, 1) : idesc_bf16_f32(128, 64, 0, 1);
      const uint32_t idesc_h = idesc_bf16_f32(128, 64, 0, 1);    // Yf or Yb: N = P, B = one state block
      const uint32_t cbase = smem_u32(smem + kOutOffC), hbase = smem_u32(smem + kOutOffH);
      int k = 0, kg = 0;
      bool ok = true;
      for (int g = blockIdx.x; g < ngroups && ok; g += gridDim.x, ++kg) {
        for (int h = 0; h < nh; ++h, ++k) {
          const int buf = k & 1, use = k >> 1, acc = k & 1;
          const uint32_t xb = smem_u32(smem + buf * kOutXBuf);
          const uint32_t ybase = tmem + 128 + acc * 192;
          // Yf (+)= C Hf^T or Yb (+)= C Hb^T from the ring slot of part q (0: Hf hi, 1: Hb hi, 2: Hf lo, 3: Hb lo)
          auto state_product = [&](int q) -> bool {
            const int u = 4 * k + q, sl = u % 3, hu = u / 3;
            if (!mbar_wait(&h_full[sl], hu & 1)) return false;
            tc_fence_after();
            const uint32_t hs = hbase + sl * 16384;
#pragma unroll
            for (int kq = 0; kq < 8; ++kq)   // K = N_state = 128
              mma_bf16_ss(ybase + 64 + (q & 1) * 64, desc_sw128(cbase + (kq >> 2) * 16384 + (kq & 3) * 32, 16, 1024),
                          desc_sw128(hs + kq * 2048, 16384, 1024), idesc_h, (q >> 1) != 0 || kq > 0);
            mma_commit(&h_empty[sl]);
            return true;
          };
          ok = mbar_wait(&y_empty[acc], (use & 1) ^ 1) && mbar_wait(&m_full[0], k & 1);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int q = 0; q < 8; ++q)   // Yd = M x, first K half (M in TMEM, 8 columns per 16 elements)
            mma_bf16_ts(ybase, tmem + q * 8, desc_sw128(xb + q * 2048, 32768, 1024), idesc_d, q > 0);
          mma_commit(&m_empty[0]);
          ok = (h > 0 || mbar_wait(c_full, kg & 1)) && state_product(0) && state_product(1);
          if (!ok) break;
          ok = mbar_wait(&m_full[1], k & 1);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int q = 8; q < 16; ++q)   // Yd, second K half
            mma_bf16_ts(ybase, tmem + q * 8, desc_sw128(xb + q * 2048, 32768, 1024), idesc_d, true);
          mma_commit(&m_empty[1]);
          mma_commit(&x_empty[buf]);
          ok = state_product(2) && state_product(3);
          if (!ok) break;
          if (h == nh - 1) mma_commit(c_empty);
          mma_commit(&y_full[acc]);
        }
      }
    }
    __syncwarp();
  } else if (warp < kOutFirstEpiWarp) {
    // ------------------------------------------------------------------------------ transform
    const int xw = warp - kOutFirstXformWarp;
    const int quad = warp & 3, half = xw >> 2;
    const int r = quad * 32 + lane;
    const uint32_t tm_row = tmem + (static_cast<uint32_t>(quad * 32) << 16) + half * 16;
    int k = 0, kg = 0;
    bool ok = true;
    for (int g = blockIdx.x; g < ngroups && ok; g += gridDim.x, ++kg) {
      const int t = g & 1;
      const int i = t * 128 + r, ib = i >> 6;
      for (int h = 0; h < nh && ok; ++h, ++k) {
        const int buf = k & 1, use = k >> 1;
        if (!wait_all(&x_full[buf], use & 1)) { ok = false; break; }
        const float* tb = reinterpret_cast<const float*>(smem + kOutOffTbl + buf * kOutTblBytes);
        const float ufi = tb[kTUf + r], ubi = tb[kTUb + r];
        const float si2 = tb[kTSi + r], sxi2 = tb[kTSx + r];
        const float* wfr = tb + kTWf + (ib - 2 * t) * 256;
        const float* wbr = tb + kTWb + (ib - 2 * t) * 256;
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
          const int hh = cb >> 1;
          if ((cb & 1) == 0) {
            if (!wait_all(&m_empty[hh], (k & 1) ^ 1)) { ok = false; break; }
            tc_fence_after();
          }
          if (h == 0 && !wait_all(&g_full[cb], kg & 1)) { ok = false; break; }
          const uint8_t* grow = smem + kOutOffG + cb * 16384 + r * 128;
          // this warp's 4 consecutive 16-byte chunks of the row (32 elements, 16 contiguous TMEM columns),
          // stored with one 16-column TMEM store
          const uint32_t tcol = tm_row + cb * 32;
          uint32_t pk[16];
          if (cb != ib && XF16) {
            // M = (G w) u in packed fp16: two multiplies per element pair
            const uint32_t uu = pack_f16x2_sat(cb < ib ? ufi : ubi, cb < ib ? ufi : ubi);
            const __half* wh = reinterpret_cast<const __half*>(tb + (cb < ib ? kTWf : kTWb)) + (ib - 2 * t) * 256 +
                               cb * 64 + half * 32;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int ch = 4 * half + c;
              const uint4 gc = *reinterpret_cast<const uint4*>(grow + ((ch ^ (r & 7)) << 4));
              const uint4 wv = *reinterpret_cast<const uint4*>(wh + c * 8);
              pk[4 * c + 0] = mul_f16x2(mul_f16x2(gc.x, wv.x), uu);
              pk[4 * c + 1] = mul_f16x2(mul_f16x2(gc.y, wv.y), uu);
              pk[4 * c + 2] = mul_f16x2(mul_f16x2(gc.z, wv.z), uu);
              pk[4 * c + 3] = mul_f16x2(mul_f16x2(gc.w, wv.w), uu);
            }
          } else if (cb != ib) {
            const float u = cb < ib ? ufi : ubi;
            const float2 uu = make_float2(u, u);
            const float* w = (cb < ib ? wfr : wbr) + cb * 64 + half * 32;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int ch = 4 * half + c;
              const uint4 gc = *reinterpret_cast<const uint4*>(grow + ((ch ^ (r & 7)) << 4));
              const float4 wa = *reinterpret_cast<const float4*>(w + c * 8);
              const float4 wc = *reinterpret_cast<const float4*>(w + c * 8 + 4);
              // the same products as g * (u * w) elementwise, two per instruction
              const float2 m0 = mul_f32x2(unpack_f16x2(gc.x), mul_f32x2(uu, make_float2(wa.x, wa.y)));
              const float2 m1 = mul_f32x2(unpack_f16x2(gc.y), mul_f32x2(uu, make_float2(wa.z, wa.w)));
              const float2 m2 = mul_f32x2(unpack_f16x2(gc.z), mul_f32x2(uu, make_float2(wc.x, wc.y)));
              const float2 m3 = mul_f32x2(unpack_f16x2(gc.w), mul_f32x2(uu, make_float2(wc.z, wc.w)));
              pk[4 * c + 0] = pack_bf16x2(m0.x, m0.y);
              pk[4 * c + 1] = pack_bf16x2(m1.x, m1.y);
              pk[4 * c + 2] = pack_bf16x2(m2.x, m2.y);
              pk[4 * c + 3] = pack_bf16x2(m3.x, m3.y);
            }
          } else {
            // one exponential per element in the log2 domain; the diagonal itself is added in fp32 in
            // the epilogue
            const float* lfr = tb + kTLf - 128 * t;
            const float* lbr = tb + kTLb - 128 * t;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int ch = 4 * half + c;
              const int j0 = cb * 64 + ch * 8;
              const uint4 gc = *reinterpret_cast<const uint4*>(grow + ((ch ^ (r & 7)) << 4));
              const float4 f0 = *reinterpret_cast<const float4*>(lfr + j0);
              const float4 f1 = *reinterpret_cast<const float4*>(lfr + j0 + 4);
              const float4 b0 = *reinterpret_cast<const float4*>(lbr + j0);
              const float4 b1 = *reinterpret_cast<const float4*>(lbr + j0 + 4);
              const float lf8[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
              const float lb8[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
              const uint32_t* gu = reinterpret_cast<const uint32_t*>(&gc);
              float m[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int jj = j0 + e;
                const float wv = ex2_approx(jj < i ? si2 + lf8[e] : lb8[e] - sxi2);
                m[e] = jj == i ? 0.f : wv;
              }
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                if (XF16) {
                  pk[4 * c + e] = mul_f16x2(gu[e], pack_f16x2_sat(m[2 * e], m[2 * e + 1]));
                } else {
                  const float2 gm = mul_f32x2(unpack_f16x2(gu[e]), make_float2(m[2 * e], m[2 * e + 1]));
                  pk[4 * c + e] = pack_bf16x2(gm.x, gm.y);
                }
              }
            }
          }
          tmem_st16(tcol, pk);
          if (h == nh - 1) {   // the group's last head has read this G slot
            __syncwarp();
            if (lane == 0) mbar_arrive(&g_empty[cb]);
          }
          if (cb & 1) {
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&m_full[hh]);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    int k = 0;
    bool ok = true;
    for (int g = blockIdx.x; g < ngroups && ok; g += gridDim.x) {
      int b, v, t;
      decode(g, b, v, t);
      const int i = t * 128 + r;
      const int len = min(kSsdQ, p.s.n - v * kSsdQ);
      const bool valid = i < len;
      const long long cidx = static_cast<long long>(b) * p.nVc + v;
      const float gdi = p.Gd[cidx * kSsdQ + i];
      const long long yrow = b * p.y_bstride + p.s.map(v * kSsdQ + (valid ? i : 0));
      // this token's x row (source row from the chunk's row table) and its decay-table entries are read
      // from global memory (L2), issued before the accumulators are ready, so that the x / table buffer
      // is released by the MMAs alone
      const int xsrc = valid ? p.crow[cidx * kSsdQ + i] : 0;
      const uint8_t* xrow = static_cast<const uint8_t*>(p.s.xv) + static_cast<long long>(xsrc) * p.s.ldxv * 2;
      for (int h = 0; h < nh; ++h, ++k) {
        const int acc = k & 1, use = k >> 1;
        const float Dh = p.Dp_b != nullptr ? 0.5f * (p.Dp[h] + p.Dp_b[h]) : p.Dp[h];
        const float* tg = p.tbl + ((cidx * nh + h) * 2 + t) * kOutTbl;
        const float ef = tg[kTEf + r], eb = tg[kTEb + r], dli = tg[kTDl + r];
        // x row of this token (packed bf16 or fp16 pairs) for the skip and diagonal terms
        uint32_t xw[32];
        if (valid) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xrow + h * kSsdP * 2) + q);
            xw[q * 4 + 0] = xv.x; xw[q * 4 + 1] = xv.y; xw[q * 4 + 2] = xv.z; xw[q * 4 + 3] = xv.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) xw[q] = 0u;
        }
        if (!wait_all(&y_full[acc], use & 1)) { ok = false; break; }
        tc_fence_after();
        const float D2 = 2.f * (Dh + (valid ? gdi * dli : 0.f));
        __nv_bfloat16* ydst = p.y + yrow * p.ldy + h * kSsdP;
        const uint32_t ybase = tmem + (static_cast<uint32_t>(quad * 32) << 16) + 128 + acc * 192;
#pragma unroll
        for (int pc = 0; pc < 4; ++pc) {   // 16 columns at a time
          uint32_t yd[16], yf[16], yb[16];
          tmem_ld16(ybase + pc * 16, yd);
          tmem_ld16(ybase + 64 + pc * 16, yf);
          tmem_ld16(ybase + 128 + pc * 16, yb);
          tmem_wait_ld();
          if (valid) {
            uint32_t ou[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 xf = XF16 ? unpack_f16x2(xw[pc * 8 + e]) : unpack_bf16x2(xw[pc * 8 + e]);
              const int k0 = 2 * e;
              const float y0 = __uint_as_float(yd[k0]) + ef * __uint_as_float(yf[k0]) +
                               eb * __uint_as_float(yb[k0]) + D2 * xf.x;
              const float y1 = __uint_as_float(yd[k0 + 1]) + ef * __uint_as_float(yf[k0 + 1]) +
                               eb * __uint_as_float(yb[k0 + 1]) + D2 * xf.y;
              ou[e] = pack_bf16x2(y0, y1);
            }
            uint4* dst = reinterpret_cast<uint4*>(ydst + pc * 16);
            dst[0] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
            dst[1] = make_uint4(ou[4], ou[5], ou[6], ou[7]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&y_empty[acc]);
      }
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
