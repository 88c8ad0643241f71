// Backward pass of the bidirectional selective scan, fp32 CUDA-core kernel for small problems (the training
// counterpart of ssd_f32_kernel).  The forward recurrence per head
//     a_t = exp(delta_t A),  h_t = a_t h_{t-1} + delta_t x_t B_t^T,  y_t = h_t C_t + D x_t
// has the adjoint state G_t = dy_t C_t^T + a_{t+1} G_{t+1}, run from the last row to the first, and
//     dx_t = delta_t G_t B_t + D dy_t,   dB_t = delta_t G_t^T x_t,   dC_t = h_t^T dy_t,
//     ddelta_t = x_t^T G_t B_t + A a_t <h_{t-1}, G_t>,   dA = sum_t delta_t a_t <h_{t-1}, G_t>,
//     dD = sum_t <x_t, dy_t>.
// Both directions of the bidirectional scan (forward over [prefix; video], backward over [prefix; video
// reversed]) receive the video rows' output gradient; prefix rows receive none.
#pragma once
#include "common.cuh"
#include "simt.cuh"

namespace mate {

// One CTA per (head, sample); thread (p, n) owns state element [p][n].  For each direction the CTA first
// reruns the forward recurrence, storing every state in hs ([L][P*N] floats for this CTA), then runs the
// adjoint from the last sequence position to the first.  Per-row gradients owned by this head (dx, ddt)
// are written by the first direction and accumulated by the second (same thread, program order); dB and
// dC are shared by all heads and accumulate with atomics into zeroed buffers; dA_log, dD and ddt_bias
// accumulate per CTA and are added once at the end.
// dy: [B][n][nh*P] (video rows); dx: [rows of x][nh*P]; dB, dC: [rows][N]; ddt: [rows][nh] (gradient of
// the raw step input dt, delta = softplus(dt + dt_bias)).
__global__ void ssd_backward_f32_kernel(SeqRows s, const float* __restrict__ dt, int lddt,
                                        const float* __restrict__ dt_bias, const float* __restrict__ A_log,
                                        const float* __restrict__ Dp, int P, int N, const float* __restrict__ dy,
                                        float* __restrict__ dx, float* __restrict__ dB, float* __restrict__ dC,
                                        float* __restrict__ ddt, float* __restrict__ ddt_bias,
                                        float* __restrict__ dA_log, float* __restrict__ dD, float* __restrict__ hs_all) {
  extern __shared__ float sh[];
  const int PN = P * N;
  float* r_hdy = sh;            // h_t[p][n] dy_t[p]          (sum over p: dC)
  float* r_gx = sh + PN;        // G[p][n] x_t[p]             (sum over p: dB / delta)
  float* r_gb = sh + 2 * PN;    // G[p][n] B_t[n]             (sum over n: dx / delta)
  float* r_hg = sh + 3 * PN;    // h_{t-1}[p][n] G[p][n]      (full sum)
  float* r_p = sh + 4 * PN;     // [3][P]: x_t[p] (G B_t)[p], row sums of r_hg, x_t[p] dy_t[p]
  const int h = blockIdx.x, b = blockIdx.y, nh = gridDim.x;
  const int tid = threadIdx.x;
  const bool active = tid < PN;
  const int p = active ? tid / N : 0, nn = active ? tid % N : 0;
  const int L = s.R + s.n;
  const float A = -expf(A_log[h]);
  const float Dh = Dp[h];
  const float bias = dt_bias[h];
  float* hs = hs_all + ((long long)b * nh + h) * (long long)L * PN;
  float acc_dA = 0.f, acc_dD = 0.f, acc_db = 0.f;   // thread 0 only
  for (int dir = 0; dir < 2; ++dir) {
    // sequence position i -> row of the inputs; video output row for i >= R
    auto seq_row = [&](int i) -> long long {
      if (i < s.R) return s.rrow(b, i);
      const int q = dir == 0 ? i - s.R : s.n - 1 - (i - s.R);
      return s.vrow(b, q);
    };
    auto video_q = [&](int i) -> int { return dir == 0 ? i - s.R : s.n - 1 - (i - s.R); };
    auto step = [&](long long row, float& dl, float& a) {
      const float v = dt[row * lddt + h] + bias;
      dl = v > 20.f ? v : log1pf(expf(v));
      a = expf(dl * A);
    };
    // forward recurrence, every state kept
    float hv = 0.f;
    for (int i = 0; i < L; ++i) {
      const long long row = seq_row(i);
      float dl, a;
      step(row, dl, a);
      if (active) {
        const float xp = (i < s.R ? static_cast<const float*>(s.xr) + row * s.ldxr
                                  : static_cast<const float*>(s.xv) + row * s.ldxv)[h * P + p];
        const float bn = (i < s.R ? static_cast<const float*>(s.br) + row * s.ldbr
                                  : static_cast<const float*>(s.bv) + row * s.ldbv)[nn];
        hv = a * hv + dl * xp * bn;
        hs[(long long)i * PN + tid] = hv;
      }
    }
    __syncthreads();
    // adjoint, last position first
    float G = 0.f, a_next = 0.f;
    for (int i = L - 1; i >= 0; --i) {
      const long long row = seq_row(i);
      float dl, a;
      step(row, dl, a);
      const bool pre = i < s.R;
      const float* xr = pre ? static_cast<const float*>(s.xr) + row * s.ldxr : static_cast<const float*>(s.xv) + row * s.ldxv;
      const float* br = pre ? static_cast<const float*>(s.br) + row * s.ldbr : static_cast<const float*>(s.bv) + row * s.ldbv;
      const float* cr = pre ? static_cast<const float*>(s.cr) + row * s.ldcr : static_cast<const float*>(s.cv) + row * s.ldcv;
      const float dyv = (!pre && active) ? dy[((long long)b * s.n + video_q(i)) * (long long)nh * P + h * P + p] : 0.f;
      float xp = 0.f;
      if (active) {
        xp = xr[h * P + p];
        G = (i + 1 < L ? a_next * G : 0.f) + dyv * cr[nn];
        const float ht = hs[(long long)i * PN + tid];
        const float hp = i > 0 ? hs[(long long)(i - 1) * PN + tid] : 0.f;
        r_hdy[tid] = ht * dyv;
        r_gx[tid] = G * xp;
        r_gb[tid] = G * br[nn];
        r_hg[tid] = hp * G;
      }
      __syncthreads();
      if (active && p == 0) {          // per n: sums over p
        float sc = 0.f, sb = 0.f;
        for (int k = 0; k < P; ++k) {
          sc += r_hdy[k * N + nn];
          sb += r_gx[k * N + nn];
        }
        atomicAdd(&dC[row * N + nn], sc);
        atomicAdd(&dB[row * N + nn], dl * sb);
      }
      if (active && nn == 0) {         // per p: sums over n
        float sg = 0.f, sh_ = 0.f;
        for (int k = 0; k < N; ++k) {
          sg += r_gb[p * N + k];
          sh_ += r_hg[p * N + k];
        }
        const float g = dl * sg + Dh * dyv;
        float* dst = (pre ? dx + row * s.ldxr : dx + row * s.ldxv) + h * P + p;
        *dst = dir == 0 ? g : *dst + g;
        r_p[p] = xp * sg;
        r_p[P + p] = sh_;
        r_p[2 * P + p] = xp * dyv;
      }
      __syncthreads();
      if (tid == 0) {
        float xgb = 0.f, hg = 0.f, xdy = 0.f;
        for (int k = 0; k < P; ++k) {
          xgb += r_p[k];
          hg += r_p[P + k];
          xdy += r_p[2 * P + k];
        }
        const float ddelta = xgb + A * a * hg;
        const float v = dt[row * lddt + h] + bias;
        const float g = ddelta / (1.f + expf(-v));      // softplus'(v) = sigmoid(v)
        float* dst = ddt + row * lddt + h;
        *dst = dir == 0 ? g : *dst + g;
        acc_dA += dl * a * hg;
        acc_dD += xdy;
        acc_db += g;
      }
      a_next = a;
      __syncthreads();
    }
  }
  if (tid == 0) {
    atomicAdd(&dA_log[h], acc_dA * A);    // A = -exp(A_log): dA/dA_log = A
    atomicAdd(&dD[h], acc_dD);
    atomicAdd(&ddt_bias[h], acc_db);
  }
}

}  // namespace mate
