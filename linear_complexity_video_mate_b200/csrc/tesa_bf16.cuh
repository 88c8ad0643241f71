// TEmporal Swin Attention on tcgen05 (news article, method section, TESA paragraph; "LinGen：基于Mamba机制
// 的线性复杂度高清长视频生成框架", 关键算法创新 / TESA): attention inside fixed 3D windows of
// wt x wh x ww = 256 tokens, with the window grid shifted by (st, sh, sw) on odd layers (Swin style:
// roll by minus the shift, partition, mask wrapped tokens from the others, roll back).
//
// Persistent: a CTA walks the (window, sample, head) items blockIdx.x, blockIdx.x + gridDim.x, ...
//   warps 0..3   loaders: the item's token rows (cyclic shift folded into the row addresses) and Swin
//                region codes into one of two row tables; Q and K rows ([256 tok][128 dim], 128B-swizzled,
//                K-major) by cp.async once the previous item's S = Q K^T has been computed; V rows (the
//                same layout, read MN-major) once the previous item's P V is done.
//   warp 4       MMA issue (lane 0): S_t = Q_t K^T for the two 128-query tiles t into TMEM columns
//                [256 t, 256 t + 256); then O_t = P_t V with P_t read from TMEM into [256 t + 128, 256 t + 256).
//   warps 5..12  softmax and output, one warp per (TMEM lane quadrant, query tile), one thread per query
//                row: exact row softmax over all 256 keys (region mask only in windows that hold several
//                wrap regions), P written in bf16 back into the row's own S columns ([256 t, 256 t + 128),
//                two keys per column, each column written after it was read); then O / rowsum to global,
//                32 columns at a time through a 2 KB transpose buffer per warp, so that each store
//                instruction writes eight whole 64-byte row segments.
// P never touches shared memory, so Q / K / V buffers are refilled while the softmax and P V of the
// current item run.
#pragma once
#include "common.cuh"

namespace mate {

struct TesaBf16Params {
  const __nv_bfloat16* qkv;  // rows b*n + raster, row stride ldq; q / k / v of head h at qcol/kcol/vcol + h*tp
  int ldq, qcol, kcol, vcol;
  __nv_bfloat16* O;          // rows b*n + raster, row stride ldo, head h at ocol + h*tp
  int ldo, ocol;
  int B, T, H, W, th;
  int wt, wh, ww;
  int st, sh, sw;            // zero when the layer is not shifted
  int shifted;
  float scale_log2;          // log2(e) / sqrt(tp)
};

__device__ __forceinline__ int tesa_region(int p, int D, int w, int s) { return p < D - w ? 0 : (p < D - s ? 1 : 2); }

constexpr int kTesaLoadWarps = 4, kTesaMmaWarp = 4, kTesaFirstSoftWarp = 5, kTesaSoftWarps = 8;
constexpr int kTesaThreads = (kTesaFirstSoftWarp + kTesaSoftWarps) * 32;   // 416

struct TesaRows {   // per item, two of them
  long long srow[256];   // global row of each window token
  int code[256];         // Swin region code of each token
  int mixed[kTesaLoadWarps];
};
constexpr uint32_t kTesaOffQ = 0, kTesaOffK = 65536, kTesaOffV = 131072, kTesaOffRows = 196608;
constexpr uint32_t kTesaOffBar = kTesaOffRows + 2 * 3328;
constexpr uint32_t kTesaOffStage = kTesaOffBar + 256;   // output transpose buffers, 2 KB per softmax warp
constexpr uint32_t kTesaSmem = kTesaOffStage + kTesaSoftWarps * 2048;
static_assert(kTesaSmem + 1024 <= 232448, "shared memory of the TESA kernel");
static_assert(sizeof(TesaRows) <= 3328, "row table size");

__global__ void __launch_bounds__(kTesaThreads, 1) tesa_bf16_kernel(const TesaBf16Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kTesaOffQ;   // [256 tok][128 dim] K-major, 64-dim blocks 32 KB apart
  uint8_t* sK = smem + kTesaOffK;
  uint8_t* sV = smem + kTesaOffV;   // same layout, used MN-major
  TesaRows* rows = reinterpret_cast<TesaRows*>(smem + kTesaOffRows);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTesaOffBar);
  uint64_t* qk_full = bars;       // 128 loader threads (cp.async arrivals)
  uint64_t* qk_empty = bars + 1;  // S MMA commit
  uint64_t* v_full = bars + 2;    // 128 loader threads
  uint64_t* v_empty = bars + 3;   // P V MMA commit
  uint64_t* tb_full = bars + 4;   // [2] 128 loader threads
  uint64_t* tb_empty = bars + 6;  // [2] 8 softmax warps
  uint64_t* s_full = bars + 8;    // S MMA commit
  uint64_t* p_full = bars + 9;    // 256 softmax threads
  uint64_t* o_full = bars + 10;   // P V MMA commit
  uint64_t* s_free = bars + 11;   // 8 softmax warps (O read: TMEM free for the next S)
  uint32_t* slot = reinterpret_cast<uint32_t*>(bars + 12);

  const int nwt = p.T / p.wt, nwh = p.H / p.wh, nww = p.W / p.ww;
  const int nwin = nwt * nwh * nww;
  const int nitems = nwin * p.B * p.th;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = p.T * p.H * p.W;

  if (threadIdx.x == 0) {
    mbar_init(qk_full, kTesaLoadWarps * 32);
    mbar_init(qk_empty, 1);
    mbar_init(v_full, kTesaLoadWarps * 32);
    mbar_init(v_empty, 1);
    for (int q = 0; q < 2; ++q) {
      mbar_init(&tb_full[q], kTesaLoadWarps * 32);
      mbar_init(&tb_empty[q], kTesaSoftWarps);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, kTesaSoftWarps * 32);
    mbar_init(o_full, 1);
    mbar_init(s_free, kTesaSoftWarps);
    mbar_fence_init();
  }
  if (warp == kTesaMmaWarp) {
    tmem_alloc(slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;

  // item -> (window, sample, head); heads innermost so that consecutive items share the window's rows
  auto decode = [&](int it, int& win, int& b, int& hd) {
    hd = it % p.th;
    const int rest = it / p.th;
    win = rest % nwin;
    b = rest / nwin;
  };

  if (warp < kTesaLoadWarps) {
    // ------------------------------------------------------------------------------ loaders
    const int lt = threadIdx.x;   // 0..127
    bool failed = false;
    int k = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++k) {
      const int tbuf = k & 1;
      int win, b, hd;
      decode(it, win, b, hd);
      const bool okt = mbar_wait(&tb_empty[tbuf], ((k >> 1) & 1) ^ 1);
      // a wait that ran out makes all loader threads leave together (a thread leaving alone would strand
      // the others at the named barrier)
      if (named_bar_any(1, kTesaLoadWarps * 32, failed || !okt)) break;
      TesaRows& rt = rows[tbuf];
      const int wi_w = win % nww, wi_h = (win / nww) % nwh, wi_t = win / (nww * nwh);
      bool differs = false;
      const int code0 = p.shifted ? tesa_region(wi_t * p.wt, p.T, p.wt, p.st) * 9 +
                                        tesa_region(wi_h * p.wh, p.H, p.wh, p.sh) * 3 +
                                        tesa_region(wi_w * p.ww, p.W, p.ww, p.sw)
                                  : 0;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        // token kk of the window (raster inside the window) in shifted coordinates -> original grid row
        const int kk = lt + 128 * u;
        const int e = kk % p.ww, c = (kk / p.ww) % p.wh, a = kk / (p.ww * p.wh);
        const int pt = wi_t * p.wt + a, ph = wi_h * p.wh + c, pw = wi_w * p.ww + e;
        const int ot = (pt + p.st) % p.T, oh = (ph + p.sh) % p.H, ow = (pw + p.sw) % p.W;
        rt.srow[kk] = static_cast<long long>(b) * n + (static_cast<long long>(ot) * p.H + oh) * p.W + ow;
        const int code = p.shifted ? (tesa_region(pt, p.T, p.wt, p.st) * 9 + tesa_region(ph, p.H, p.wh, p.sh) * 3 +
                                      tesa_region(pw, p.W, p.ww, p.sw))
                                   : 0;
        rt.code[kk] = code;
        differs = differs || code != code0;
      }
      const bool wmixed = __any_sync(0xffffffffu, differs);
      if (lane == 0) rt.mixed[warp] = wmixed ? 1 : 0;
      named_bar_sync(1, kTesaLoadWarps * 32);   // the row table is complete
      mbar_arrive(&tb_full[tbuf]);
      const int qc = p.qcol + hd * 128, kc = p.kcol + hd * 128, vc = p.vcol + hd * 128;
      // Q and K, once the previous item's S is computed
      const bool okq = mbar_wait(qk_empty, (k & 1) ^ 1);
      failed = failed || !okq;
      if (okq) {
        for (int itc = lt; itc < 256 * 16; itc += kTesaLoadWarps * 32) {
          const int r = itc >> 4, ch = itc & 15;
          const __nv_bfloat16* row = p.qkv + rt.srow[r] * p.ldq;
          const uint32_t off = sw128_kmajor_offset(r, ch * 8, 32768);
          cp_async16(sQ + off, row + qc + ch * 8);
          cp_async16(sK + off, row + kc + ch * 8);
        }
        cp_async_arrive(qk_full);
      }
      // V, once the previous item's P V is done
      const bool okv = okq && mbar_wait(v_empty, (k & 1) ^ 1);
      failed = failed || !okv;
      if (okv) {
        for (int itc = lt; itc < 256 * 16; itc += kTesaLoadWarps * 32) {
          const int r = itc >> 4, ch = itc & 15;
          cp_async16(sV + sw128_kmajor_offset(r, ch * 8, 32768), p.qkv + rt.srow[r] * p.ldq + vc + ch * 8);
        }
        cp_async_arrive(v_full);
      }
    }
    cp_async_wait<0>();
  } else if (warp == kTesaMmaWarp) {
    // ------------------------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 256, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t q0 = smem_u32(sQ), k0 = smem_u32(sK), v0 = smem_u32(sV);
      int k = 0;
      for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++k) {
        if (!mbar_wait(qk_full, k & 1) || !mbar_wait(s_free, (k & 1) ^ 1)) break;
        fence_proxy_async();   // cp.async writes (generic proxy) -> tensor-core reads
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const uint32_t off = (s & 3) * 32;
            mma_bf16_ss(tmem + t * 256, desc_sw128(q0 + (s >> 2) * 32768 + t * 16384 + off, 16, 1024),
                        desc_sw128(k0 + (s >> 2) * 32768 + off, 16, 1024), idesc_s, s > 0);
          }
        mma_commit(s_full);
        mma_commit(qk_empty);
        if (!mbar_wait(p_full, k & 1) || !mbar_wait(v_full, k & 1)) break;
        fence_proxy_async();
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int s = 0; s < 16; ++s)   // O_t = P_t V: P_t from TMEM (8 columns per 16 keys), V MN-major
            mma_bf16_ts(tmem + t * 256 + 128, tmem + t * 256 + s * 8, desc_sw128(v0 + s * 2048, 32768, 1024),
                        idesc_o, s > 0);
        mma_commit(o_full);
        mma_commit(v_empty);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------------------ softmax and output
    const int sw = warp - kTesaFirstSoftWarp;
    const int quad = warp & 3, t = sw >> 2;
    const int r = quad * 32 + lane;   // row inside the query tile
    const int i = t * 128 + r;        // query token of the window
    const uint32_t srow_t = tmem + (static_cast<uint32_t>(quad * 32) << 16) + t * 256;
    int k = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++k) {
      const int tbuf = k & 1;
      int win, b, hd;
      decode(it, win, b, hd);
      if (__any_sync(0xffffffffu, !mbar_wait(&tb_full[tbuf], (k >> 1) & 1))) break;
      const TesaRows& rt = rows[tbuf];
      bool has_mask = false;
#pragma unroll
      for (int w = 0; w < kTesaLoadWarps; ++w) has_mask = has_mask || rt.mixed[w] != 0;
      const int myc = rt.code[i];
      if (__any_sync(0xffffffffu, !mbar_wait(s_full, k & 1))) break;
      tc_fence_after();
      // two 32-column TMEM loads in flight per wait
      float mx = -INFINITY;
#pragma unroll 1
      for (int c0 = 0; c0 < 256; c0 += 64) {
        uint32_t v[32], w[32];
        tmem_ld32(srow_t + c0, v);
        tmem_ld32(srow_t + c0 + 32, w);
        tmem_wait_ld();
        if (has_mask) {
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            if (rt.code[c0 + u] == myc) mx = fmaxf(mx, __uint_as_float(v[u]));
            if (rt.code[c0 + 32 + u] == myc) mx = fmaxf(mx, __uint_as_float(w[u]));
          }
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) mx = fmaxf(mx, fmaxf(__uint_as_float(v[u]), __uint_as_float(w[u])));
        }
      }
      const float mxs = mx * p.scale_log2;
      float sum = 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < 256; c0 += 64) {
        uint32_t v[64];
        tmem_ld32(srow_t + c0, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(srow_t + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
        uint32_t pk[32];
#pragma unroll
        for (int u = 0; u < 64; u += 2) {
          float e0 = ex2_approx(fmaf(__uint_as_float(v[u]), p.scale_log2, -mxs));
          float e1 = ex2_approx(fmaf(__uint_as_float(v[u + 1]), p.scale_log2, -mxs));
          if (has_mask) {
            if (rt.code[c0 + u] != myc) e0 = 0.f;
            if (rt.code[c0 + u + 1] != myc) e1 = 0.f;
          }
          sum += e0 + e1;
          pk[u / 2] = pack_bf16x2(e0, e1);
        }
        // columns [c0 / 2, c0 / 2 + 32) were read already (they lie below c0 + 64)
        tmem_st16(srow_t + c0 / 2, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
        tmem_st16(srow_t + c0 / 2 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
      const float inv = 1.f / sum;
      if (__any_sync(0xffffffffu, !mbar_wait(o_full, k & 1))) break;
      tc_fence_after();
      // this warp's 32 rows x 32 columns at a time: 16-byte chunk c of row r at position c ^ ((r >> 1) & 3)
      // (conflict-free writes and reads), then four lanes per row segment
      uint4* stg = reinterpret_cast<uint4*>(smem + kTesaOffStage + sw * 2048);
      const long long* srw = rt.srow + t * 128 + quad * 32;
      __nv_bfloat16* ob = p.O + p.ocol + hd * 128;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(srow_t + 128 + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 pk;
          pk.x = pack_bf16x2(__uint_as_float(v[q * 8 + 0]) * inv, __uint_as_float(v[q * 8 + 1]) * inv);
          pk.y = pack_bf16x2(__uint_as_float(v[q * 8 + 2]) * inv, __uint_as_float(v[q * 8 + 3]) * inv);
          pk.z = pack_bf16x2(__uint_as_float(v[q * 8 + 4]) * inv, __uint_as_float(v[q * 8 + 5]) * inv);
          pk.w = pack_bf16x2(__uint_as_float(v[q * 8 + 6]) * inv, __uint_as_float(v[q * 8 + 7]) * inv);
          stg[lane * 4 + (q ^ ((lane >> 1) & 3))] = pk;
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int rr = u * 8 + (lane >> 2), q = lane & 3;
          reinterpret_cast<uint4*>(ob + srw[rr] * p.ldo + c0)[q] = stg[rr * 4 + (q ^ ((rr >> 1) & 3))];
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(s_free);
        mbar_arrive(&tb_empty[tbuf]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kTesaMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mate
