// Backward pass of TEmporal Swin Attention on tcgen05 (training; the pages give the forward computation
// only: news article, method section, TESA paragraph; "LinGen：基于Mamba机制的线性复杂度高清长视频生成框架",
// 关键算法创新 / TESA).  Per window and head, with S = Q K^T / sqrt(tp) (Swin region mask in windows that
// hold several wrap regions), P = softmax(S) row-wise and O = P V, the gradients follow by the chain rule:
//   dV = P^T dO,   dP = dO V^T,   dS = P (dP - delta),  delta_i = sum_j P_ij dP_ij = dO_i . O_i,
//   dQ = dS K / sqrt(tp),   dK = dS^T Q / sqrt(tp).
// Two kernels, one CTA per (window, sample, head, 128-row block), everything of an item on chip:
//   tesa_bwd_dq_kernel    query block qb: S and dP against all 256 keys (TMEM columns [0, 256) and
//                         [256, 512)), the exact row statistics (max, sum) and delta, then dS (bf16, into
//                         the V buffer once dP is done) and dQ = dS K.  Writes per query L2 = log2 of the
//                         softmax normaliser (in units of the scaled scores) and delta for the second kernel.
//   tesa_bwd_dkdv_kernel  key block kb: for the two query tiles in turn, S and dP against the block's 128
//                         keys, P and dS from the stored statistics (bf16 into shared memory, read MN-major
//                         as the A operand), and dV += P^T dO, dK += dS^T Q in TMEM columns [256, 512).
// Precision: the products run on fp16 operands.  q, k, v and dO are bf16 in memory and convert to fp16
// exactly on the way into shared memory; P and dS are rounded to fp16 (8 times finer than bf16: dQ and dK
// sum dS terms that cancel, since every row of dS sums to zero, so their relative error is amplified).
// Values beyond the fp16 range saturate at +-65504.
// One thread issues the MMAs; all 8 warps do the elementwise work (two warps per TMEM lane quadrant, one
// column half each).  Bounded waits as everywhere in the library: a wait that runs out flags the device
// status word and the CTA skips the rest of its item.
#pragma once
#include "common.cuh"
#include "tesa_bf16.cuh"

namespace mate {

struct TesaBwdParams {
  const __nv_bfloat16* qkv;  // [B n][ldq]: q | k | v, head h at qcol/kcol/vcol + h tp
  int ldq, qcol, kcol, vcol;
  const __nv_bfloat16* O;    // forward output [B n][ldo], head h at ocol + h tp
  const __nv_bfloat16* dO;   // its gradient, same layout
  int ldo, ocol;
  __nv_bfloat16* dqkv;       // [B n][ldg]: dq | dk | dv at gq/gk/gv + h tp
  int ldg, gq, gk, gv;
  float* stats;              // [items][256][2]: L2 (log2 of the row normaliser), delta
  int B, T, H, W, th;
  int wt, wh, ww;
  int st, sh, sw;
  int shifted;
  float scale_log2;          // log2(e) / sqrt(tp)
  float scale;               // 1 / sqrt(tp)
};

constexpr int kTesaBwdThreads = 256;

struct TesaBwdRows {
  int srow[256];            // global row of each window token (shifted coordinates -> grid)
  unsigned char code[256];  // Swin region code of each token
  float red[2][128];        // partial row reductions of the two column halves
  float L2[256];            // per query: log2 normaliser, delta
  float delta[256];
  int mixed;
};

// The 8 bf16 values of a 16-byte shared-memory chunk converted to fp16 in place (exact inside the fp16
// range).  Operands arrive by cp.async (all of an item's copies in flight at once); each thread converts
// the chunks it copied itself, after its own copies have landed.
__device__ __forceinline__ void tesa_bwd_to_f16(uint8_t* p) {
  uint4 v = *reinterpret_cast<const uint4*>(p);
  float2 f = unpack_bf16x2(v.x); v.x = pack_f16x2_sat(f.x, f.y);
  f = unpack_bf16x2(v.y); v.y = pack_f16x2_sat(f.x, f.y);
  f = unpack_bf16x2(v.z); v.z = pack_f16x2_sat(f.x, f.y);
  f = unpack_bf16x2(v.w); v.w = pack_f16x2_sat(f.x, f.y);
  *reinterpret_cast<uint4*>(p) = v;
}

// Row table of an item (all 256 window tokens); returns whether the window mixes wrap regions.
__device__ __forceinline__ bool tesa_bwd_rows(const TesaBwdParams& p, int item, TesaBwdRows& rt, int& hd) {
  const int nwt = p.T / p.wt, nwh = p.H / p.wh, nww = p.W / p.ww;
  const int nwin = nwt * nwh * nww;
  hd = item % p.th;
  const int rest = item / p.th;
  const int win = rest % nwin, b = rest / nwin;
  const int wi_w = win % nww, wi_h = (win / nww) % nwh, wi_t = win / (nww * nwh);
  const int kk = threadIdx.x;   // one token per thread
  const int e = kk % p.ww, c = (kk / p.ww) % p.wh, a = kk / (p.ww * p.wh);
  const int pt = wi_t * p.wt + a, ph = wi_h * p.wh + c, pw = wi_w * p.ww + e;
  const int ot = (pt + p.st) % p.T, oh = (ph + p.sh) % p.H, ow = (pw + p.sw) % p.W;
  const int n = p.T * p.H * p.W;
  rt.srow[kk] = b * n + (ot * p.H + oh) * p.W + ow;
  const int code = p.shifted ? tesa_region(pt, p.T, p.wt, p.st) * 9 + tesa_region(ph, p.H, p.wh, p.sh) * 3 +
                                   tesa_region(pw, p.W, p.ww, p.sw)
                             : 0;
  rt.code[kk] = static_cast<unsigned char>(code);
  const int code0 = p.shifted ? tesa_region(wi_t * p.wt, p.T, p.wt, p.st) * 9 +
                                    tesa_region(wi_h * p.wh, p.H, p.wh, p.sh) * 3 +
                                    tesa_region(wi_w * p.ww, p.W, p.ww, p.sw)
                              : 0;
  return __syncthreads_or(code != code0) != 0;
}

// ---------------------------------------------------------------------------------------------------
// dQ, row statistics and delta.  grid (items, 2 query blocks), 256 threads.
// ---------------------------------------------------------------------------------------------------
constexpr uint32_t kBdqK = 0, kBdqV = 65536, kBdqQ = 131072, kBdqDO = 163840, kBdqRows = 196608;
constexpr uint32_t kBdqBar = kBdqRows + ((sizeof(TesaBwdRows) + 15) / 16) * 16;
constexpr uint32_t kBdqSmem = kBdqBar + 64;

__global__ void __launch_bounds__(kTesaBwdThreads, 1) tesa_bwd_dq_kernel(const TesaBwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + kBdqK;     // [256 keys][128 d], 64-d blocks 32 KB apart
  uint8_t* sV = smem + kBdqV;     // same; after dP: dS [128 q][256 keys] K-major, 64-key blocks 16 KB apart
  uint8_t* sQ = smem + kBdqQ;     // [128 q][128 d], 64-d blocks 16 KB apart
  uint8_t* sDO = smem + kBdqDO;   // same
  TesaBwdRows& rt = *reinterpret_cast<TesaBwdRows*>(smem + kBdqRows);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kBdqBar);
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 1);
  const int item = blockIdx.x, qb = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3, hf = warp >> 2;
  const int r = quad * 32 + lane;   // query row inside the block
  const int qi = qb * 128 + r;      // query token of the window

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  int hd;
  const bool has_mask = tesa_bwd_rows(p, item, rt, hd);   // ends with a block barrier
  const int qc = p.qcol + hd * 128, kc = p.kcol + hd * 128, vc = p.vcol + hd * 128;
  for (int it = threadIdx.x; it < 256 * 16; it += kTesaBwdThreads) {
    const int rr = it >> 4, ch = it & 15;
    const __nv_bfloat16* row = p.qkv + static_cast<long long>(rt.srow[rr]) * p.ldq;
    const uint32_t off = sw128_kmajor_offset(rr, ch * 8, 32768);
    cp_async16(sK + off, row + kc + ch * 8);
    cp_async16(sV + off, row + vc + ch * 8);
  }
  for (int it = threadIdx.x; it < 128 * 16; it += kTesaBwdThreads) {
    const int rr = it >> 4, ch = it & 15;
    const long long g = rt.srow[qb * 128 + rr];
    const uint32_t off = sw128_kmajor_offset(rr, ch * 8, 16384);
    cp_async16(sQ + off, p.qkv + g * p.ldq + qc + ch * 8);
    cp_async16(sDO + off, p.dO + g * p.ldo + p.ocol + hd * 128 + ch * 8);
  }
  cp_async_commit();
  cp_async_wait<0>();
  for (int it = threadIdx.x; it < 256 * 16; it += kTesaBwdThreads) {
    const uint32_t off = sw128_kmajor_offset(it >> 4, (it & 15) * 8, 32768);
    tesa_bwd_to_f16(sK + off);
    tesa_bwd_to_f16(sV + off);
  }
  for (int it = threadIdx.x; it < 128 * 16; it += kTesaBwdThreads) {
    const uint32_t off = sw128_kmajor_offset(it >> 4, (it & 15) * 8, 16384);
    tesa_bwd_to_f16(sQ + off);
    tesa_bwd_to_f16(sDO + off);
  }
  fence_proxy_async();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t q0 = smem_u32(sQ), k0 = smem_u32(sK), v0 = smem_u32(sV), o0 = smem_u32(sDO);
  if (threadIdx.x == 0) {
    const uint32_t idesc = idesc_f16_f32(128, 256, 0, 0);
#pragma unroll
    for (int s = 0; s < 8; ++s) {   // S = Q K^T and dP = dO V^T, K = 128 dims
      const uint32_t off = (s & 3) * 32;
      mma_bf16_ss(tmem, desc_sw128(q0 + (s >> 2) * 16384 + off, 16, 1024),
                  desc_sw128(k0 + (s >> 2) * 32768 + off, 16, 1024), idesc, s > 0);
      mma_bf16_ss(tmem + 256, desc_sw128(o0 + (s >> 2) * 16384 + off, 16, 1024),
                  desc_sw128(v0 + (s >> 2) * 32768 + off, 16, 1024), idesc, s > 0);
    }
    mma_commit(bar);
  }
  bool ok = !__syncthreads_or(!mbar_wait(bar, 0));
  tc_fence_after();
  const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const int myc = rt.code[qi];
  if (ok) {
    // row maximum over this thread's column half, then over both
    float mx = -INFINITY;
    for (int c0 = hf * 128; c0 < hf * 128 + 128; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(trow + c0, v);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 32; ++u)
        if (!has_mask || rt.code[c0 + u] == myc) mx = fmaxf(mx, __uint_as_float(v[u]));
    }
    rt.red[hf][r] = mx;
    __syncthreads();
    mx = fmaxf(rt.red[0][r], rt.red[1][r]);
    __syncthreads();
    const float mxs = mx * p.scale_log2;
    float sum = 0.f;
    for (int c0 = hf * 128; c0 < hf * 128 + 128; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(trow + c0, v);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 32; ++u)
        if (!has_mask || rt.code[c0 + u] == myc) sum += ex2_approx(fmaf(__uint_as_float(v[u]), p.scale_log2, -mxs));
    }
    // delta_i = dO_i . O_i over this thread's half of the dimensions (dO from shared memory, O from global)
    float dl = 0.f;
    const __nv_bfloat16* orow = p.O + static_cast<long long>(rt.srow[qi]) * p.ldo + p.ocol + hd * 128 + hf * 64;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint4 ov = __ldg(reinterpret_cast<const uint4*>(orow) + q);
      const uint4 dv = *reinterpret_cast<const uint4*>(sDO + sw128_kmajor_offset(r, hf * 64 + q * 8, 16384));
      const uint32_t* ow = reinterpret_cast<const uint32_t*>(&ov);
      const uint32_t* dw = reinterpret_cast<const uint32_t*>(&dv);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 a = unpack_bf16x2(ow[e]), g = unpack_f16x2(dw[e]);
        dl = fmaf(a.x, g.x, fmaf(a.y, g.y, dl));
      }
    }
    rt.red[hf][r] = sum;
    __syncthreads();
    sum = rt.red[0][r] + rt.red[1][r];
    const float L2 = mxs + __log2f(sum);
    __syncthreads();
    rt.red[hf][r] = dl;
    __syncthreads();
    const float delta = rt.red[0][r] + rt.red[1][r];
    if (hf == 0) {
      float* sp = p.stats + (static_cast<long long>(item) * 256 + qi) * 2;
      sp[0] = L2;
      sp[1] = delta;
    }
    // dS = P (dP - delta) in fp16, K-major [128 q][256 keys] in the V buffer (dP has been computed)
    for (int c0 = hf * 128; c0 < hf * 128 + 128; c0 += 32) {
      uint32_t s[32], g[32];
      tmem_ld32(trow + c0, s);
      tmem_ld32(trow + 256 + c0, g);
      tmem_wait_ld();
#pragma unroll
      for (int u8 = 0; u8 < 32; u8 += 8) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int u = u8 + 2 * e;
          float p0 = ex2_approx(fmaf(__uint_as_float(s[u]), p.scale_log2, -L2));
          float p1 = ex2_approx(fmaf(__uint_as_float(s[u + 1]), p.scale_log2, -L2));
          if (has_mask) {
            if (rt.code[c0 + u] != myc) p0 = 0.f;
            if (rt.code[c0 + u + 1] != myc) p1 = 0.f;
          }
          pk[e] = pack_f16x2_sat(p0 * (__uint_as_float(g[u]) - delta), p1 * (__uint_as_float(g[u + 1]) - delta));
        }
        *reinterpret_cast<uint4*>(sV + sw128_kmajor_offset(r, c0 + u8, 16384)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  if (ok && threadIdx.x == 0) {
    tc_fence_after();
    const uint32_t idesc = idesc_f16_f32(128, 128, 0, 1);
#pragma unroll
    for (int s = 0; s < 16; ++s)   // dQ = dS K: A = dS K-major, B = K rows read MN-major (N = dims)
      mma_bf16_ss(tmem, desc_sw128(v0 + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024), desc_sw128(k0 + s * 2048, 32768, 1024),
                  idesc, s > 0);
    mma_commit(bar);
  }
  ok = ok && !__syncthreads_or(!mbar_wait(bar, 1));
  tc_fence_after();
  if (ok) {
    __nv_bfloat16* drow = p.dqkv + static_cast<long long>(rt.srow[qi]) * p.ldg + p.gq + hd * 128 + hf * 64;
    for (int c0 = 0; c0 < 64; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(trow + hf * 64 + c0, v);
      tmem_wait_ld();
      uint4* dst = reinterpret_cast<uint4*>(drow + c0);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        dst[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]) * p.scale, __uint_as_float(v[8 * q + 1]) * p.scale),
                            pack_bf16x2(__uint_as_float(v[8 * q + 2]) * p.scale, __uint_as_float(v[8 * q + 3]) * p.scale),
                            pack_bf16x2(__uint_as_float(v[8 * q + 4]) * p.scale, __uint_as_float(v[8 * q + 5]) * p.scale),
                            pack_bf16x2(__uint_as_float(v[8 * q + 6]) * p.scale, __uint_as_float(v[8 * q + 7]) * p.scale));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------------------
// dK and dV.  grid (items, 2 key blocks), 256 threads; needs the statistics of tesa_bwd_dq_kernel.
// ---------------------------------------------------------------------------------------------------
constexpr uint32_t kBkvK = 0, kBkvV = 32768, kBkvQ = 65536, kBkvDO = 98304, kBkvP = 131072, kBkvS = 163840;
constexpr uint32_t kBkvRows = 196608;
constexpr uint32_t kBkvBar = kBkvRows + ((sizeof(TesaBwdRows) + 15) / 16) * 16;
constexpr uint32_t kBkvSmem = kBkvBar + 64;

__global__ void __launch_bounds__(kTesaBwdThreads, 1) tesa_bwd_dkdv_kernel(const TesaBwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + kBkvK;     // [128 keys][128 d], 64-d blocks 16 KB apart
  uint8_t* sV = smem + kBkvV;
  uint8_t* sQ = smem + kBkvQ;     // [128 q][128 d] of the current query tile
  uint8_t* sDO = smem + kBkvDO;
  uint8_t* sP = smem + kBkvP;     // [128 q][128 keys], 64-key blocks 16 KB apart: P read MN-major (M = keys)
  uint8_t* sdS = smem + kBkvS;    // same for dS
  TesaBwdRows& rt = *reinterpret_cast<TesaBwdRows*>(smem + kBkvRows);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kBkvBar);
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 1);
  const int item = blockIdx.x, kb = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3, hf = warp >> 2;
  const int r = quad * 32 + lane;

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  int hd;
  const bool has_mask = tesa_bwd_rows(p, item, rt, hd);
  const int qc = p.qcol + hd * 128, kc = p.kcol + hd * 128, vc = p.vcol + hd * 128;
  {
    const float* sp = p.stats + (static_cast<long long>(item) * 256 + threadIdx.x) * 2;
    rt.L2[threadIdx.x] = sp[0];
    rt.delta[threadIdx.x] = sp[1];
  }
  for (int it = threadIdx.x; it < 128 * 16; it += kTesaBwdThreads) {
    const int rr = it >> 4, ch = it & 15;
    const __nv_bfloat16* row = p.qkv + static_cast<long long>(rt.srow[kb * 128 + rr]) * p.ldq;
    const uint32_t off = sw128_kmajor_offset(rr, ch * 8, 16384);
    cp_async16(sK + off, row + kc + ch * 8);
    cp_async16(sV + off, row + vc + ch * 8);
  }
  cp_async_commit();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const uint32_t q0 = smem_u32(sQ), k0 = smem_u32(sK), v0 = smem_u32(sV), o0 = smem_u32(sDO);
  const uint32_t p0 = smem_u32(sP), s0 = smem_u32(sdS);
  bool ok = true;
  for (int t = 0; t < 2 && ok; ++t) {
    for (int it = threadIdx.x; it < 128 * 16; it += kTesaBwdThreads) {
      const int rr = it >> 4, ch = it & 15;
      const long long g = rt.srow[t * 128 + rr];
      const uint32_t off = sw128_kmajor_offset(rr, ch * 8, 16384);
      cp_async16(sQ + off, p.qkv + g * p.ldq + qc + ch * 8);
      cp_async16(sDO + off, p.dO + g * p.ldo + p.ocol + hd * 128 + ch * 8);
    }
    cp_async_commit();
    cp_async_wait<0>();
    for (int it = threadIdx.x; it < 128 * 16; it += kTesaBwdThreads) {
      const uint32_t off = sw128_kmajor_offset(it >> 4, (it & 15) * 8, 16384);
      tesa_bwd_to_f16(sQ + off);
      tesa_bwd_to_f16(sDO + off);
      if (t == 0) {   // the key block's K and V (copied by this thread in the same pattern) on the first tile
        tesa_bwd_to_f16(sK + off);
        tesa_bwd_to_f16(sV + off);
      }
    }
    fence_proxy_async();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_f16_f32(128, 128, 0, 0);
#pragma unroll
      for (int s = 0; s < 8; ++s) {   // S = Q_t K_kb^T, dP = dO_t V_kb^T
        const uint32_t off = (s >> 2) * 16384 + (s & 3) * 32;
        mma_bf16_ss(tmem, desc_sw128(q0 + off, 16, 1024), desc_sw128(k0 + off, 16, 1024), idesc, s > 0);
        mma_bf16_ss(tmem + 128, desc_sw128(o0 + off, 16, 1024), desc_sw128(v0 + off, 16, 1024), idesc, s > 0);
      }
      mma_commit(bar);
    }
    ok = !__syncthreads_or(!mbar_wait(bar, (2 * t) & 1));
    tc_fence_after();
    if (ok) {
      // P and dS of query row r (tile t) against this thread's half of the block's keys
      const int qi = t * 128 + r;
      const int myc = rt.code[qi];
      const float L2 = rt.L2[qi], delta = rt.delta[qi];
      for (int c0 = hf * 64; c0 < hf * 64 + 64; c0 += 32) {
        uint32_t s[32], g[32];
        tmem_ld32(trow + c0, s);
        tmem_ld32(trow + 128 + c0, g);
        tmem_wait_ld();
#pragma unroll
        for (int u8 = 0; u8 < 32; u8 += 8) {
          uint32_t pp[4], pd[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int u = u8 + 2 * e;
            float a0 = ex2_approx(fmaf(__uint_as_float(s[u]), p.scale_log2, -L2));
            float a1 = ex2_approx(fmaf(__uint_as_float(s[u + 1]), p.scale_log2, -L2));
            if (has_mask) {
              if (rt.code[kb * 128 + c0 + u] != myc) a0 = 0.f;
              if (rt.code[kb * 128 + c0 + u + 1] != myc) a1 = 0.f;
            }
            pp[e] = pack_f16x2_sat(a0, a1);
            pd[e] = pack_f16x2_sat(a0 * (__uint_as_float(g[u]) - delta), a1 * (__uint_as_float(g[u + 1]) - delta));
          }
          const uint32_t off = sw128_mnmajor_offset(r, c0 + u8, 16384);
          *reinterpret_cast<uint4*>(sP + off) = make_uint4(pp[0], pp[1], pp[2], pp[3]);
          *reinterpret_cast<uint4*>(sdS + off) = make_uint4(pd[0], pd[1], pd[2], pd[3]);
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (ok && threadIdx.x == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_f16_f32(128, 128, 1, 1);
#pragma unroll
      for (int s = 0; s < 8; ++s) {   // dV += P^T dO_t, dK += dS^T Q_t: K = the tile's 128 queries
        mma_bf16_ss(tmem + 256, desc_sw128(p0 + s * 2048, 16384, 1024), desc_sw128(o0 + s * 2048, 16384, 1024), idesc,
                    t > 0 || s > 0);
        mma_bf16_ss(tmem + 384, desc_sw128(s0 + s * 2048, 16384, 1024), desc_sw128(q0 + s * 2048, 16384, 1024), idesc,
                    t > 0 || s > 0);
      }
      mma_commit(bar);
    }
    ok = ok && !__syncthreads_or(!mbar_wait(bar, (2 * t + 1) & 1));
    tc_fence_after();
  }
  if (ok) {
    // row r of the accumulators = key kb * 128 + r; this thread writes one half of the dimensions
    const long long g = rt.srow[kb * 128 + r];
    __nv_bfloat16* dv = p.dqkv + g * p.ldg + p.gv + hd * 128 + hf * 64;
    __nv_bfloat16* dk = p.dqkv + g * p.ldg + p.gk + hd * 128 + hf * 64;
    for (int c0 = 0; c0 < 64; c0 += 32) {
      uint32_t a[32], b[32];
      tmem_ld32(trow + 256 + hf * 64 + c0, a);
      tmem_ld32(trow + 384 + hf * 64 + c0, b);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        reinterpret_cast<uint4*>(dv + c0)[q] =
            make_uint4(pack_bf16x2(__uint_as_float(a[8 * q]), __uint_as_float(a[8 * q + 1])),
                       pack_bf16x2(__uint_as_float(a[8 * q + 2]), __uint_as_float(a[8 * q + 3])),
                       pack_bf16x2(__uint_as_float(a[8 * q + 4]), __uint_as_float(a[8 * q + 5])),
                       pack_bf16x2(__uint_as_float(a[8 * q + 6]), __uint_as_float(a[8 * q + 7])));
        reinterpret_cast<uint4*>(dk + c0)[q] =
            make_uint4(pack_bf16x2(__uint_as_float(b[8 * q]) * p.scale, __uint_as_float(b[8 * q + 1]) * p.scale),
                       pack_bf16x2(__uint_as_float(b[8 * q + 2]) * p.scale, __uint_as_float(b[8 * q + 3]) * p.scale),
                       pack_bf16x2(__uint_as_float(b[8 * q + 4]) * p.scale, __uint_as_float(b[8 * q + 5]) * p.scale),
                       pack_bf16x2(__uint_as_float(b[8 * q + 6]) * p.scale, __uint_as_float(b[8 * q + 7]) * p.scale));
      }
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
