// CUDA-core kernels of the MATE block:
//   * Rotary Major Scan row gather/scatter and review-token pooling (both dtypes, HBM-bound copies);
//   * the fp32 path of the block (projections, selective scan, window attention) for small fp32 blocks,
//     where fp32 accuracy matters more than tensor-core throughput;
//   * small helpers (weight packing, softplus of raw step sizes).
#pragma once
#include "common.cuh"
#include "gemm_bf16.cuh"

namespace mate {

// ---------------------------------------------------------------------------------------------------
// Rotary Major Scan: dst row (b, i) = src row (b, map(i)); map = scan->raster (permute) or
// raster->scan (unpermute).  One warp per destination row, 16-byte vectors; rows are contiguous
// d-vectors so both the gather reads and the writes are full-row coalesced.
// ---------------------------------------------------------------------------------------------------
__global__ void rms_gather_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, long long total_rows,
                                       int n, int vec_per_row, int T, int H, int W, int order, int inverse) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < total_rows;
       row += warps) {
    const long long b = row / n;
    const int i = static_cast<int>(row - b * n);
    const int j = inverse ? raster_to_scan(i, T, H, W, order) : scan_to_raster(i, T, H, W, order);
    const uint4* s = src + (b * n + j) * vec_per_row;
    uint4* d = dst + row * vec_per_row;
    for (int v = lane; v < vec_per_row; v += 32) d[v] = __ldg(s + v);
  }
}

// Rows stored in scan order (src, row stride ld_src vectors) back to grid order (dst, row stride ld_dst
// vectors): dst row b*n + r = src row b*n + raster_to_scan(r).  One warp per row, 16-byte vectors.
__global__ void scan_rows_to_grid_kernel(const uint4* __restrict__ src, long long ld_src, uint4* __restrict__ dst,
                                         long long ld_dst, int vec_per_row, long long total_rows, int n, int T, int H,
                                         int W, int order) {
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < total_rows;
       row += warps) {
    const long long b = row / n;
    const int r = static_cast<int>(row - b * n);
    const uint4* s = src + (b * n + raster_to_scan(r, T, H, W, order)) * ld_src;
    uint4* d = dst + row * ld_dst;
    for (int v = lane; v < vec_per_row; v += 32) d[v] = __ldg(s + v);
  }
}

// ---------------------------------------------------------------------------------------------------
// Review tokens: block mean of X over each cell of the Tr x 4 x 4 pooling grid, written in scan order
// of that grid.  One CTA per review token; each thread owns one 16-byte vector of channels.
// ---------------------------------------------------------------------------------------------------
template <typename T_>
__global__ void review_pool_kernel(const T_* __restrict__ X, T_* __restrict__ Rv, int R, int T, int H, int W,
                                   int d, int order) {
  constexpr int kVec = 16 / sizeof(T_);
  const int b = blockIdx.y;
  const int q = blockIdx.x;          // scan position on the pooled grid
  const int Tr = R / 16;
  const int ft = T / Tr, fh = H / 4, fw = W / 4;
  const int cell = scan_to_raster(q, Tr, 4, 4, order);
  const int ct = cell / 16, ch = (cell / 4) % 4, cw = cell % 4;
  const float inv = 1.0f / static_cast<float>(ft * fh * fw);
  for (int c0 = threadIdx.x * kVec; c0 < d; c0 += blockDim.x * kVec) {
    float acc[kVec];
#pragma unroll
    for (int e = 0; e < kVec; ++e) acc[e] = 0.f;
    for (int a = 0; a < ft; ++a)
      for (int bb = 0; bb < fh; ++bb) {
        const long long rowbase = ((long long)b * T * H + (long long)(ct * ft + a) * H + (ch * fh + bb)) * W + cw * fw;
        for (int c = 0; c < fw; ++c) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(X + (rowbase + c) * d + c0));
          const T_* e8 = reinterpret_cast<const T_*>(&v);
#pragma unroll
          for (int e = 0; e < kVec; ++e) acc[e] += static_cast<float>(e8[e]);
        }
      }
    uint4 o;
    T_* o8 = reinterpret_cast<T_*>(&o);
#pragma unroll
    for (int e = 0; e < kVec; ++e) o8[e] = static_cast<T_>(acc[e] * inv);
    *reinterpret_cast<uint4*>(Rv + ((long long)b * R + q) * d + c0) = o;
  }
}

// ---------------------------------------------------------------------------------------------------
// Weight packing: dst rows [row0, row0 + rows) of a [*, ldd] matrix <- src [rows, cols] at column col0.
// ---------------------------------------------------------------------------------------------------
__global__ void copy_block_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int rows, int vec_cols,
                                  int ld_dst_vec, int row0, int col0_vec) {
  const long long total = (long long)rows * vec_cols;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / vec_cols;
    const int c = static_cast<int>(i - r * vec_cols);
    dst[(row0 + r) * ld_dst_vec + col0_vec + c] = __ldg(src + i);
  }
}

// delta = softplus(dt + dt_bias) for [rows, nh] raw step sizes.
// out[row][c] = softplus(dt[row][c] + bias[c]); with bias2, rows of out hold 2 nh values and
// out[row][nh + c] = softplus(dt[row][c] + bias2[c]).
__global__ void softplus_kernel(const float* __restrict__ dt, const float* __restrict__ bias,
                                const float* __restrict__ bias2, float* __restrict__ out, long long total, int nh) {
  const int ld = bias2 != nullptr ? 2 * nh : nh;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / nh;
    const int c = static_cast<int>(i - row * nh);
    const float v = dt[i] + bias[c];
    out[row * ld + c] = v > 20.f ? v : log1pf(expf(v));
    if (bias2 != nullptr) {
      const float v2 = dt[i] + bias2[c];
      out[row * ld + nh + c] = v2 > 20.f ? v2 : log1pf(expf(v2));
    }
  }
}

// ---------------------------------------------------------------------------------------------------
// Self-test of the timeout report: one thread waits on a fresh mbarrier that nothing arrives at, polling
// at most max_polls times, then records MATE_DEV_TIMEOUT in the device status word and returns, as every
// bounded wait of the library does when it runs out.
// ---------------------------------------------------------------------------------------------------
__global__ void wait_timeout_selftest_kernel(unsigned max_polls) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(&bar, 1);
  mbar_fence_init();
  for (unsigned i = 0; i < max_polls; ++i) {
    if (mbar_try_wait(&bar, 0)) return;   // phase 0 never completes: no thread arrives
    __nanosleep(64);
  }
  flag_status(MATE_DEV_TIMEOUT);
}

// ---------------------------------------------------------------------------------------------------
// fp32 path
// ---------------------------------------------------------------------------------------------------

// C[M, N] (ldc) = A[M, K] (lda) * B[N, K]^T (ldb); optional softplus side output of columns
// [dt_col0, dt_col0 + dt_cols) into delta[M, ld_delta].  64 x 64 tiles, 4 x 4 outputs per thread.
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A, int lda, const float* __restrict__ Bm,
                                                       int ldb, float* __restrict__ C, int ldc, int M, int N, int K,
                                                       float* __restrict__ delta, int ld_delta, int dt_col0,
                                                       int dt_cols, const float* __restrict__ dt_bias,
                                                       const float* __restrict__ dt_bias2, const GemmEpilogue ep) {
  __shared__ float As[16][65];
  __shared__ float Bs[16][65];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      const int r = i / 16, k = i % 16;
      As[k][r] = (m0 + r < M && k0 + k < K) ? A[(long long)(m0 + r) * lda + k0 + k] : 0.f;
      Bs[k][r] = (n0 + r < N && k0 + k < K) ? Bm[(long long)(n0 + r) * ldb + k0 + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k)
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(As[k][ty * 4 + a], Bs[k][tx * 4 + c], acc[a][c]);
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int r = m0 + ty * 4 + a;
    if (r >= M) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int col = n0 + tx * 4 + c;
      if (col >= N) continue;
      float v = acc[a][c];
      if (ep.bias != nullptr) v += ep.bias[col];
      if (ep.act == 1) v = gelu_tanh_f<false>(v);
      if (ep.resid != nullptr)
        v = static_cast<const float*>(ep.resid)[(long long)r * ep.ld_resid + col] +
            (ep.gate != nullptr ? ep.gate[(long long)(r / ep.gate_rows) * ep.ld_gate + col] : 1.f) * v;
      C[(long long)r * ldc + col] = v;
      if (delta != nullptr && col >= dt_col0 && col < dt_col0 + dt_cols) {
        const float v = acc[a][c] + dt_bias[col - dt_col0];
        delta[(long long)r * ld_delta + col - dt_col0] = v > 20.f ? v : log1pf(expf(v));
        if (dt_bias2 != nullptr) {   // the backward scan's step size, dt_cols columns further on
          const float v2 = acc[a][c] + dt_bias2[col - dt_col0];
          delta[(long long)r * ld_delta + dt_cols + col - dt_col0] = v2 > 20.f ? v2 : log1pf(expf(v2));
        }
      }
    }
  }
}

// Sequence row access shared by the scan kernels.  Position i of sample b's sequence is a prefix row
// (i < R: row b*r_bstride + r_off + i of the prefix arrays) or the video row of scan position q = i - R
// (row b*v_bstride + v_off + map(q) of the video arrays, map = scan_to_raster for order >= 0, identity
// for order < 0).  x / B / C / delta have their own base pointers and row strides (elements).
struct SeqRows {
  const void* xv; const void* bv; const void* cv; const float* dv;
  const void* xr; const void* br; const void* cr; const float* dr;
  int ldxv, ldbv, ldcv, lddv;
  int ldxr, ldbr, ldcr, lddr;
  long long v_bstride, v_off, r_bstride, r_off;
  int n, R, T, H, W;
  int db_off;    // column offset of the backward direction's delta in the delta rows (0: shared delta)
  int order;     // scan order of the video input rows (row of scan position q: scan_to_raster(q)); -1: identity
  int y_order;   // scan order of the output rows (y of scan position q goes to row map(q)); -1: identity
  int x_f16 = 0; // bf16 tensor-core scan: the x rows are fp16 (1) or bf16 (0); B and C rows are bf16
  __host__ __device__ __forceinline__ int map(int q) const {
    return y_order < 0 ? q : scan_to_raster(q, T, H, W, y_order);
  }
  __host__ __device__ __forceinline__ int in_map(int q) const {
    return order < 0 ? q : scan_to_raster(q, T, H, W, order);
  }
  __host__ __device__ __forceinline__ long long vrow(int b, int q) const { return b * v_bstride + v_off + in_map(q); }
  __host__ __device__ __forceinline__ long long rrow(int b, int i) const { return b * r_bstride + r_off + i; }
};

// fp32 selective scan, one CTA per (head, sample); thread (p, n) owns state element h[p][n].  Runs the
// recurrence over [prefix; video] and then over [prefix; video reversed], adding both video outputs
// into y at row b*y_bstride + map(q) (so the video rows land back in grid order when map is a scan).
__global__ void ssd_f32_kernel(SeqRows s, const float* __restrict__ A_log, const float* __restrict__ Dp,
                               const float* __restrict__ A_log_b, const float* __restrict__ Dp_b, int P, int N,
                               float* __restrict__ y, int ldy, long long y_bstride) {
  extern __shared__ float red[];  // [P*N]
  const int h = blockIdx.x, b = blockIdx.y;
  const int p = threadIdx.x / N, nn = threadIdx.x % N;
  const bool active = threadIdx.x < P * N;
  const int L = s.R + s.n;
  for (int dir = 0; dir < 2; ++dir) {
    // the backward scan may have its own parameters and its delta at column offset db_off
    const float A = -expf((dir == 1 && A_log_b != nullptr ? A_log_b : A_log)[h]);
    const float Dh = (dir == 1 && Dp_b != nullptr ? Dp_b : Dp)[h];
    const int dcol = (dir == 1 ? s.db_off : 0) + h;
    float hs = 0.f;
    for (int i = 0; i < L; ++i) {
      const float *xrow, *brow, *crow;
      float dl;
      long long yrow = -1;
      if (i < s.R) {
        const long long r = s.rrow(b, i);
        xrow = static_cast<const float*>(s.xr) + r * s.ldxr;
        brow = static_cast<const float*>(s.br) + r * s.ldbr;
        crow = static_cast<const float*>(s.cr) + r * s.ldcr;
        dl = s.dr[r * s.lddr + dcol];
      } else {
        const int q = dir == 0 ? i - s.R : s.n - 1 - (i - s.R);
        const long long r = s.vrow(b, q);
        yrow = b * y_bstride + s.map(q);
        xrow = static_cast<const float*>(s.xv) + r * s.ldxv;
        brow = static_cast<const float*>(s.bv) + r * s.ldbv;
        crow = static_cast<const float*>(s.cv) + r * s.ldcv;
        dl = s.dv[r * s.lddv + dcol];
      }
      float xp = 0.f;
      if (active) {
        xp = xrow[h * P + p];
        hs = expf(dl * A) * hs + dl * xp * brow[nn];
        red[threadIdx.x] = hs * crow[nn];
      }
      __syncthreads();
      if (active && nn == 0 && yrow >= 0) {
        float acc = Dh * xp;
        for (int k = 0; k < N; ++k) acc += red[p * N + k];
        float* dst = y + yrow * ldy + h * P + p;
        *dst = (dir == 0 ? 0.f : *dst) + acc;
      }
      __syncthreads();
    }
  }
}

// Swin region of shifted coordinate p on an axis (length D, window w, shift s).
__device__ __forceinline__ int swin_region(int p, int D, int w, int s) { return p < D - w ? 0 : (p < D - s ? 1 : 2); }

// fp32 window attention: one warp per (query token, head, sample); online softmax over the window.
__global__ void tesa_f32_kernel(const float* __restrict__ qkv, int ldq, int qcol, int kcol, int vcol,
                                float* __restrict__ O, int ldo, int ocol, int T, int H, int W, int th, int tp, int wt,
                                int wh, int ww, int st, int sh, int sw, int shifted) {
  const int lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int n = T * H * W;
  if (gw >= (long long)n * th) return;
  const int b = blockIdx.y;
  const int hd = static_cast<int>(gw % th);
  const int r = static_cast<int>(gw / th);
  const int ow = r % W, oh = (r / W) % H, ot = r / (W * H);
  if (!shifted) { st = sh = sw = 0; }
  const int pt = (ot - st + T) % T, ph = (oh - sh + H) % H, pw = (ow - sw + W) % W;
  const int rq = shifted ? (swin_region(pt, T, wt, st) * 9 + swin_region(ph, H, wh, sh) * 3 + swin_region(pw, W, ww, sw)) : 0;
  const int t0 = (pt / wt) * wt, h0 = (ph / wh) * wh, w0 = (pw / ww) * ww;
  const float* qrow = qkv + ((long long)b * n + r) * ldq + qcol + hd * tp;
  const float scale = rsqrtf(static_cast<float>(tp));
  float qv[4], acc[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int dd = lane + 32 * e;
    qv[e] = dd < tp ? qrow[dd] * scale : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int a = 0; a < wt; ++a)
    for (int c = 0; c < wh; ++c)
      for (int e = 0; e < ww; ++e) {
        const int kt = t0 + a, kh = h0 + c, kw = w0 + e;
        if (shifted) {
          const int rk = swin_region(kt, T, wt, st) * 9 + swin_region(kh, H, wh, sh) * 3 + swin_region(kw, W, ww, sw);
          if (rk != rq) continue;
        }
        const long long krow = (long long)b * n + (((kt + st) % T) * H + (kh + sh) % H) * W + (kw + sw) % W;
        const float* kp = qkv + krow * ldq + kcol + hd * tp;
        const float* vp = qkv + krow * ldq + vcol + hd * tp;
        float dot = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int dd = lane + 32 * u;
          if (dd < tp) dot += qv[u] * kp[dd];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        const float mn = fmaxf(m, dot);
        const float corr = expf(m - mn);
        const float pexp = expf(dot - mn);
        l = l * corr + pexp;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int dd = lane + 32 * u;
          acc[u] = acc[u] * corr + (dd < tp ? pexp * vp[dd] : 0.f);
        }
        m = mn;
      }
  float* orow = O + ((long long)b * n + r) * ldo + ocol + hd * tp;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int dd = lane + 32 * u;
    if (dd < tp) orow[dd] = acc[u] / l;
  }
}

}  // namespace mate
