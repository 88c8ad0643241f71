// The DiT block around the MATE token mixer.  The pages say MATE replaces a DiT's self-attention and keeps
// the rest of the block ("Towards High-Resolution Minute-Length Text-to-Video Generation with Linear
// Computational Complexity", abstract; LinGen news article, method section) without describing that rest;
// the block here is the standard DiT block with adaLN-Zero conditioning:
//   [shift_a, scale_a, gate_a, shift_m, scale_m, gate_m] = silu(c) W_ada^T + b_ada       (per sample)
//   X1  = X  + gate_a * MATE(LN(X)  (1 + scale_a) + shift_a)
//   Out = X1 + gate_m * (W2 gelu_tanh(W1 (LN(X1) (1 + scale_m) + shift_m) + b1) + b2)
// with layer norms without affine parameters (eps 1e-6).  The two GEMMs of the MLP and the MATE projections
// run on the tensor-core GEMM with epilogue transforms (bias, GELU, gated residual); the kernels here are
// the small modulation product and the layer norm + modulation pass.
#pragma once
#include "common.cuh"

namespace mate {

constexpr float kDitLnEps = 1e-6f;

// mod[b][j] = b_ada[j] + sum_k silu(c[b][k]) W_ada[j][k], j < 6 d.  One warp per output; fp32 arithmetic.
template <typename T>
__global__ void __launch_bounds__(256) ada_modulation_kernel(const float* __restrict__ c, int dc,
                                                             const T* __restrict__ W_ada,
                                                             const float* __restrict__ b_ada, float* __restrict__ mod,
                                                             int nout, int B) {
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<long long>(B) * nout) return;
  const int b = static_cast<int>(wid / nout), j = static_cast<int>(wid % nout);
  const float* cb = c + static_cast<long long>(b) * dc;
  const T* wr = W_ada + static_cast<long long>(j) * dc;
  float acc = 0.f;
  for (int k = lane; k < dc; k += 32) {
    const float v = cb[k];
    acc = fmaf(v / (1.f + expf(-v)), static_cast<float>(wr[k]), acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) mod[wid] = acc + b_ada[j];
}

// h[row] = LN(x[row]) (1 + scale[s]) + shift[s] for rows of sample s = row / rows_per_sample; shift and
// scale are rows of the modulation [B][6][d] at mod + s * 6 d.  One warp per row, the row in registers
// (two passes over the registers: mean, then the mean square of the deviations); V elements per 16-byte
// vector, d <= 2048.
template <typename T, int V>
__global__ void __launch_bounds__(256) ln_modulate_kernel(const T* __restrict__ x, T* __restrict__ h, long long rows,
                                                          int d, long long rows_per_sample,
                                                          const float* __restrict__ shift,
                                                          const float* __restrict__ scale) {
  constexpr int kMaxVec = 64 / V;   // 2048 elements over 32 lanes
  const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const T* xr = x + row * d;
  float v[kMaxVec][V];
  float sum = 0.f;
#pragma unroll
  for (int q = 0; q < kMaxVec; ++q) {
    const int c0 = (q * 32 + lane) * V;
    if (c0 < d) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(xr + c0));
      const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
      for (int i = 0; i < V; ++i) {
        v[q][i] = static_cast<float>(e[i]);
        sum += v[q][i];
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / d;
  float sq = 0.f;
#pragma unroll
  for (int q = 0; q < kMaxVec; ++q) {
    const int c0 = (q * 32 + lane) * V;
    if (c0 < d) {
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const float t = v[q][i] - mean;
        sq = fmaf(t, t, sq);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  const float rstd = rsqrtf(sq / d + kDitLnEps);
  const long long s = row / rows_per_sample;
  const float* sh = shift + s * 6 * d;
  const float* sc = scale + s * 6 * d;
  T* hr = h + row * d;
#pragma unroll
  for (int q = 0; q < kMaxVec; ++q) {
    const int c0 = (q * 32 + lane) * V;
    if (c0 < d) {
      // shift and scale of these V channels: V / 4 sixteen-byte loads each (the modulation rows are
      // 16-byte aligned: 6 d floats per sample, d a multiple of 8)
      float scv[V], shv[V];
#pragma unroll
      for (int i = 0; i < V; i += 4) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(sc + c0 + i));
        const float4 b = __ldg(reinterpret_cast<const float4*>(sh + c0 + i));
        scv[i] = a.x; scv[i + 1] = a.y; scv[i + 2] = a.z; scv[i + 3] = a.w;
        shv[i] = b.x; shv[i + 1] = b.y; shv[i + 2] = b.z; shv[i + 3] = b.w;
      }
      uint4 u;
      T* e = reinterpret_cast<T*>(&u);
#pragma unroll
      for (int i = 0; i < V; ++i) e[i] = static_cast<T>(fmaf((v[q][i] - mean) * rstd, 1.f + scv[i], shv[i]));
      *reinterpret_cast<uint4*>(hr + c0) = u;
    }
  }
}

}  // namespace mate
