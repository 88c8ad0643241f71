// TEmporal Swin Attention on tcgen05 (news article, method section, TESA paragraph; "LinGen：基于Mamba机制
// 的线性复杂度高清长视频生成框架", 关键算法创新 / TESA): attention inside fixed 3D windows of
// wt x wh x ww = 256 tokens, with the window grid shifted by (st, sh, sw) on odd layers (Swin style:
// roll by minus the shift, partition, mask wrapped tokens from the others, roll back).
//
// One CTA per (window, sample, head), 16 warps.  The window's 256 token rows are gathered (with the
// cyclic shift folded into the row addresses) straight into 128B-swizzled tiles:
//   Q [256 tok][128 dim] K-major, K [256 tok][128 dim] K-major, V [256 key][128 dim] MN-major.
// S_t = Q_t K^T for the two 128-query tiles t goes to TMEM columns [256 t, 256 t + 256).  The warps read
// their rows of S_t, apply the region mask (only windows that hold wrapped tokens have one) and the exact
// row softmax (all 256 keys are on chip, no online rescaling), write P_t in bf16 over the dead Q (t = 0) /
// K (t = 1) tiles, and O_t = P_t V lands in TMEM columns [256 t, 256 t + 128); rows are divided by their
// sums on the way out.
#pragma once
#include "common.cuh"

namespace mate {

struct TesaBf16Params {
  const __nv_bfloat16* qkv;  // rows b*n + raster, row stride ldq; q / k / v of head h at qcol/kcol/vcol + h*tp
  int ldq, qcol, kcol, vcol;
  __nv_bfloat16* O;          // rows b*n + raster, row stride ldo, head h at ocol + h*tp
  int ldo, ocol;
  int T, H, W, th;
  int wt, wh, ww;
  int st, sh, sw;            // zero when the layer is not shifted
  int shifted;
  float scale_log2;          // log2(e) / sqrt(tp)
};

__device__ __forceinline__ int tesa_region(int p, int D, int w, int s) { return p < D - w ? 0 : (p < D - s ? 1 : 2); }

constexpr int kTesaThreads = 512;

// 16 warps: warp w reads TMEM lane quadrant w%4 of query tile t = (w/4)%2 and key half w/8 (softmax),
// then output-dim half w/8 (epilogue).  Row max and row sum are combined across the two halves through
// shared memory.
__global__ void __launch_bounds__(kTesaThreads, 1) tesa_bf16_kernel(const TesaBf16Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;            // Q, later P_0 ([128][256] K-major, K blocks 16 KB apart)
  uint8_t* sK = smem + 65536;    // K, later P_1
  uint8_t* sV = smem + 131072;   // V MN-major, 64-dim blocks 32 KB apart
  long long* srow = reinterpret_cast<long long*>(smem + 196608);   // [256] global row of each window token
  int* scode = reinterpret_cast<int*>(srow + 256);                 // [256] Swin region code
  float* red = reinterpret_cast<float*>(scode + 256);              // [2][256] partial row max, then row sum
  int* mixed = reinterpret_cast<int*>(red + 512);
  uint64_t* bar = reinterpret_cast<uint64_t*>(mixed + 2);          // [2]
  uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 2);

  const int nwh = p.H / p.wh, nww = p.W / p.ww;
  const int win = blockIdx.x, b = blockIdx.y, hd = blockIdx.z;
  const int wi_w = win % nww, wi_h = (win / nww) % nwh, wi_t = win / (nww * nwh);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int n = p.T * p.H * p.W;

  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    mbar_fence_init();
    *mixed = 0;
  }
  if (warp == 0) tmem_alloc(slot, 512);
  __syncthreads();
  if (tid < 256) {
    // token k of the window (raster inside the window) in shifted coordinates -> original grid row
    const int k = tid;
    const int e = k % p.ww, c = (k / p.ww) % p.wh, a = k / (p.ww * p.wh);
    const int pt = wi_t * p.wt + a, ph = wi_h * p.wh + c, pw = wi_w * p.ww + e;
    const int ot = (pt + p.st) % p.T, oh = (ph + p.sh) % p.H, ow = (pw + p.sw) % p.W;
    srow[k] = static_cast<long long>(b) * n + (static_cast<long long>(ot) * p.H + oh) * p.W + ow;
    const int code = p.shifted ? (tesa_region(pt, p.T, p.wt, p.st) * 9 + tesa_region(ph, p.H, p.wh, p.sh) * 3 +
                                  tesa_region(pw, p.W, p.ww, p.sw))
                               : 0;
    scode[k] = code;
  }
  __syncthreads();
  if (tid < 256 && scode[tid] != scode[0]) atomicOr(mixed, 1);   // the window holds several wrap regions
  const int qc = p.qcol + hd * 128, kc = p.kcol + hd * 128, vc = p.vcol + hd * 128;
  // Q and K first (one group), V second: V keeps arriving while the scores are computed
  for (int it = tid; it < 256 * 16; it += kTesaThreads) {
    const int r = it >> 4, ch = it & 15;
    const __nv_bfloat16* row = p.qkv + srow[r] * p.ldq;
    cp_async16(sQ + sw128_kmajor_offset(r, ch * 8, 32768), row + qc + ch * 8);
    cp_async16(sK + sw128_kmajor_offset(r, ch * 8, 32768), row + kc + ch * 8);
  }
  cp_async_commit();
  for (int it = tid; it < 256 * 16; it += kTesaThreads) {
    const int r = it >> 4, ch = it & 15;
    cp_async16(sV + sw128_mnmajor_offset(r, ch * 8, 32768), p.qkv + srow[r] * p.ldq + vc + ch * 8);
  }
  cp_async_commit();
  cp_async_wait<1>();
  fence_proxy_async();
  __syncthreads();   // also publishes *mixed
  tc_fence_after();
  const uint32_t tmem = *slot;

  if (tid == 0) {
    const uint32_t idesc = idesc_bf16_f32(128, 256, 0, 0);
    const uint32_t q0 = smem_u32(sQ), k0 = smem_u32(sK);
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t off = (s & 3) * 32;
        mma_bf16_ss(tmem + t * 256, desc_sw128(q0 + (s >> 2) * 32768 + t * 16384 + off, 16, 1024),
                    desc_sw128(k0 + (s >> 2) * 32768 + off, 16, 1024), idesc, s > 0);
      }
    mma_commit(&bar[0]);
  }
  const bool has_mask = *mixed != 0;
  mbar_wait(&bar[0], 0);
  tc_fence_after();

  const int quad = warp & 3, t = (warp >> 2) & 1, half = warp >> 3;
  const int r = quad * 32 + lane;        // row inside the query tile
  const int i = t * 128 + r;             // query token of the window
  const uint32_t sbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) + t * 256 + half * 128;
  const int myc = scode[i];
  float mx = -INFINITY;
  for (int c0 = 0; c0 < 128; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(sbase + c0, v);
    tmem_wait_ld();
    if (has_mask) {
#pragma unroll
      for (int u = 0; u < 32; ++u)
        if (scode[half * 128 + c0 + u] == myc) mx = fmaxf(mx, __uint_as_float(v[u]));
    } else {
#pragma unroll
      for (int u = 0; u < 32; ++u) mx = fmaxf(mx, __uint_as_float(v[u]));
    }
  }
  red[half * 256 + i] = mx;
  __syncthreads();
  mx = fmaxf(red[i], red[256 + i]);
  const float mxs = mx * p.scale_log2;
  float sum = 0.f;
  uint8_t* sP = t == 0 ? sQ : sK;
  for (int c0 = 0; c0 < 128; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(sbase + c0, v);
    tmem_wait_ld();
    uint32_t pk[16];
#pragma unroll
    for (int u = 0; u < 32; u += 2) {
      float e0 = ex2_approx(fmaf(__uint_as_float(v[u]), p.scale_log2, -mxs));
      float e1 = ex2_approx(fmaf(__uint_as_float(v[u + 1]), p.scale_log2, -mxs));
      if (has_mask) {
        if (scode[half * 128 + c0 + u] != myc) e0 = 0.f;
        if (scode[half * 128 + c0 + u + 1] != myc) e1 = 0.f;
      }
      sum += e0 + e1;
      pk[u / 2] = pack_bf16x2(e0, e1);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      *reinterpret_cast<uint4*>(sP + sw128_kmajor_offset(r, half * 128 + c0 + q * 8, 16384)) =
          make_uint4(pk[q * 4 + 0], pk[q * 4 + 1], pk[q * 4 + 2], pk[q * 4 + 3]);
  }
  __syncthreads();   // everyone has read red[] (row max) before it is reused for the sums
  red[half * 256 + i] = sum;
  cp_async_wait<0>();   // V
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 1);
    const uint32_t v0 = smem_u32(sV);
    for (int tt = 0; tt < 2; ++tt) {
      const uint32_t p0 = smem_u32(tt == 0 ? sQ : sK);
#pragma unroll 4
      for (int s = 0; s < 16; ++s)
        mma_bf16_ss(tmem + tt * 256, desc_sw128(p0 + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                    desc_sw128(v0 + s * 2048, 32768, 1024), idesc, s > 0);
    }
    mma_commit(&bar[1]);
  }
  const float inv = 1.f / (red[i] + red[256 + i]);
  mbar_wait(&bar[1], 0);
  tc_fence_after();
  __nv_bfloat16* orow = p.O + srow[i] * p.ldo + p.ocol + hd * 128 + half * 64;
  for (int c0 = 0; c0 < 64; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + t * 256 + half * 64 + c0, v);
    tmem_wait_ld();
    uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 pk;
      pk.x = pack_bf16x2(__uint_as_float(v[q * 8 + 0]) * inv, __uint_as_float(v[q * 8 + 1]) * inv);
      pk.y = pack_bf16x2(__uint_as_float(v[q * 8 + 2]) * inv, __uint_as_float(v[q * 8 + 3]) * inv);
      pk.z = pack_bf16x2(__uint_as_float(v[q * 8 + 4]) * inv, __uint_as_float(v[q * 8 + 5]) * inv);
      pk.w = pack_bf16x2(__uint_as_float(v[q * 8 + 6]) * inv, __uint_as_float(v[q * 8 + 7]) * inv);
      dst[q] = pk;
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
