// Persistent tcgen05 GEMM for the MATE block's projections: C[M, N] = A[M, K] * B[N, K]^T.
//
// Used for the MA in-projection fused with the TESA qkv projection (one GEMM over [W_in; W_qkv]) and for
// the MA out-projection fused with the TESA output projection and the branch sum (one GEMM over
// [y | O] x [W_out | W_o]^T, so Out = MA + TE falls out of the K reduction).  The projections are the
// in/out maps around the bidirectional Mamba2 block and the attention (abstract: MATE = MA + TE).
//
// Design (clusters of 2 CTAs, one CTA per SM, 6 warps each; see the two-SM section below):
//   warp 0      TMA producer: A and B tiles (BK = 64, 128-byte swizzle) into an S-stage ring;
//   warp 1      MMA issuer (leader CTA): 256 x BN x 16 tcgen05.mma.cta_group::2 into one of two TMEM
//               accumulators;
//   warps 2..9  epilogue: tcgen05.ld the finished accumulator, convert, store; the other accumulator
//               is being filled meanwhile.  Two warps per TMEM lane quadrant, one column half each, so
//               that a tile's epilogue (bias, GELU, residual, 256 columns) keeps up with a short
//               (K = 1024) main loop.  Each warp's 32 rows x 32 columns go through a 2 KB transpose
//               buffer, so that every store instruction writes eight whole 64-byte row segments.
// Optional epilogue side output: columns [dt_col0, dt_col0 + dt_cols) also produce
// delta = softplus(acc + dt_bias) in fp32 (the Mamba2 step size).  Optional epilogue transforms
// (GemmEpilogue) serve the DiT block around MATE: bias + GELU for the MLP's first layer, bias and a gated
// residual for the MLP's second layer and for the token mixer's output.
#pragma once
#include "common.cuh"

namespace mate {

// Transforms of a projection's accumulator before it is stored, applied in this order:
//   v = acc + bias[col]                               (bias: [N] fp32; null: none)
//   v = gelu_tanh(v)                                  (act == 1)
//   v = resid[row][col] + gate[row / gate_rows][col] v (resid: the residual stream, the output's element
//                                                      type; gate [M / gate_rows][ld_gate] fp32, null: 1)
struct GemmEpilogue {
  const float* bias = nullptr;
  int act = 0;
  const void* resid = nullptr;
  long long ld_resid = 0;
  const float* gate = nullptr;
  int ld_gate = 0;
  int gate_rows = 1;
};

// GELU in its tanh form, v/2 (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))); `fast` takes tanh from the
// special-function unit (relative error about 2^-11, below a bf16 rounding), otherwise from tanhf.
template <bool fast>
__device__ __forceinline__ float gelu_tanh_f(float v) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * v, v * v, v);
  float t;
  if (fast) asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(u));
  else t = tanhf(u);
  return 0.5f * v * (1.f + t);
}

struct GemmParams {
  int M, N, K;
  int bn;            // tile N (multiple of 16, <= 256)
  int num_n_tiles;   // ceil(N / bn)
  int num_tiles;     // ceil(M / 128) * num_n_tiles
  int stages;
  __nv_bfloat16* C;  // [M, ldc]
  int ldc;
  float* delta;      // optional [M, ld_delta]
  int ld_delta;
  int dt_col0, dt_cols;
  const float* dt_bias;
  const float* dt_bias2;   // optional: a second side output softplus(acc + dt_bias2) at column offset dt_cols
  GemmEpilogue ep;
  int f16_cols;      // columns [0, f16_cols) are stored as fp16 (saturating), the rest as bf16; a multiple of 32
};

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kGemmEpiWarps = 8;
constexpr int kGemmThreads = (2 + kGemmEpiWarps) * 32;   // 320

__host__ __device__ inline uint32_t gemm_stage_bytes(int bn) { return kGemmBM * 128 + bn * 128; }

__device__ __forceinline__ float softplus_f(float v) { return v > 20.f ? v : log1pf(__expf(v)); }

// ---------------------------------------------------------------------------------------------------
// Two-SM variant: a cluster of 2 CTAs computes a 256 x BN tile with tcgen05.mma.cta_group::2.  Each CTA
// loads its own 128 rows of A and BN/2 rows of B (TMA, no multicast), so the pair moves 25% fewer
// operand bytes per FLOP from L2 than two independent 128 x BN tiles and each stage is smaller (deeper
// ring).  The leader CTA (rank 0) issues the MMAs; the stage barriers that gate operand reuse live in
// both CTAs, the "operands landed" barriers only in the leader.  Each CTA's TMEM holds its 128 rows of
// the accumulator (two buffers of up to 256 columns) and each CTA runs its own epilogue.
// ---------------------------------------------------------------------------------------------------
__host__ __device__ inline uint32_t gemm_pair_stage_bytes(int bn) { return 128 * 128 + (bn / 2) * 128; }
constexpr uint32_t kGemmStageOut = kGemmEpiWarps * 2048;   // epilogue transpose buffers, after the barriers

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t stage_bytes = gemm_pair_stage_bytes(p.bn);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.stages * stage_bytes);
  uint64_t* full = bars;                  // leader only: operands of both CTAs landed
  uint64_t* empty = bars + p.stages;      // both CTAs: the pair MMAs are done with this stage
  uint64_t* tfull = bars + 2 * p.stages;  // both CTAs: accumulator ready
  uint64_t* tempty = tfull + 2;           // leader only: both CTAs' epilogues drained the accumulator
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nk = p.K / kGemmBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kGemmEpiWarps);  // the epilogue warps of both CTAs
    }
    mbar_fence_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any cross-CTA arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int tile = pair; tile < p.num_tiles && ok; tile += npairs) {
        const int mb = tile / p.num_n_tiles, nb = tile % p.num_n_tiles;
        // the pair MMA takes B rows [0, n_mma/2) from each CTA: CTA 1 holds tile columns from n_mma/2 on
        const int n_mma = min(p.bn, (p.N - nb * p.bn + 15) & ~15);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) { ok = false; break; }
          uint8_t* sa = smem + stage * stage_bytes;
          const uint32_t full_leader = map_to_cta(&full[stage], 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * stage_bytes);
          tma_load_2d_pair(&tmA, full_leader, sa, kb * kGemmBK, mb * 256 + rank * 128);
          tma_load_2d_pair(&tmB, full_leader, sa + 128 * 128, kb * kGemmBK, nb * p.bn + rank * (n_mma / 2));
          if (++stage == (uint32_t)p.stages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      uint32_t stage = 0, phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < p.num_tiles && ok; tile += npairs, ++it) {
        const int acc = it & 1;
        const uint32_t acc_par = (it >> 1) & 1;
        // the last column tile of a ragged N only multiplies the columns it has (rounded up to 16)
        const int nb = tile % p.num_n_tiles;
        const int n_mma = min(p.bn, (p.N - nb * p.bn + 15) & ~15);
        const uint32_t idesc = idesc_bf16_f32(256, n_mma, 0, 0);
        if (!mbar_wait(&tempty[acc], acc_par ^ 1)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * stage_bytes);
          const uint32_t sb = sa + 128 * 128;
#pragma unroll
          for (int k = 0; k < kGemmBK / 16; ++k)
            mma_bf16_pair(d_tmem, desc_sw128(sa + k * 32, 16, 1024), desc_sw128(sb + k * 32, 16, 1024), idesc,
                          (kb | k) != 0);
          mma_commit_pair(map_to_cta(&empty[stage], 0));
          mma_commit_pair(map_to_cta(&empty[stage], 1));
          if (++stage == (uint32_t)p.stages) { stage = 0; phase ^= 1; }
        }
        mma_commit_pair(map_to_cta(&tfull[acc], 0));
        mma_commit_pair(map_to_cta(&tfull[acc], 1));
      }
    }
  } else {
    // epilogue warps 2..9 -> TMEM lane quadrants 2, 3, 0, 1, 2, 3, 0, 1 of this CTA's 128 rows; warps 2..5
    // take the first 128 columns of a tile, warps 6..9 the rest
    const int quad = warp & 3;
    const int chalf = (warp - 2) >> 2;
    const bool has_ep = p.ep.bias != nullptr || p.ep.act != 0 || p.ep.resid != nullptr;
    int it = 0;
    for (int tile = pair; tile < p.num_tiles; tile += npairs, ++it) {
      const int mb = tile / p.num_n_tiles, nb = tile % p.num_n_tiles;
      const int acc = it & 1;
      const uint32_t acc_par = (it >> 1) & 1;
      if (!mbar_wait(&tfull[acc], acc_par)) break;
      tc_fence_after();
      const int row0 = mb * 256 + rank * 128 + quad * 32;   // this warp's first row
      const int row = row0 + lane;
      const bool row_ok = row < p.M;
      __nv_bfloat16* crow = p.C + static_cast<size_t>(row) * p.ldc;
      // 32 rows x 16-byte chunks c at position c ^ ((row >> 1) & 3): conflict-free writes and reads
      uint4* stg = reinterpret_cast<uint4*>(smem + p.stages * stage_bytes + 256) + (warp - 2) * 128;
      const int col_end = min(p.N, nb * p.bn + p.bn);
      const int c_hi = min(col_end - nb * p.bn, chalf * 128 + 128);
      for (int c0 = chalf * 128; c0 < c_hi; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * 256 + c0, r);
        tmem_wait_ld();
        const int col0 = nb * p.bn + c0;
        if (col0 >= col_end) continue;                 // the same for the whole warp
        const bool full32 = col0 + 32 <= col_end;      // the same for the whole warp
        // a full slice is stored by the whole warp together (rows past M are dropped at the store);
        // a ragged one row by row
        if (!full32 && !row_ok) continue;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (has_ep) {
          const GemmEpilogue& e = p.ep;
          if (e.bias != nullptr) {
            if (full32) {   // 32 consecutive columns: eight 16-byte loads (bias 16-byte aligned, col0 % 32 == 0)
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 b4 = __ldg(reinterpret_cast<const float4*>(e.bias + col0) + q);
                v[4 * q] += b4.x; v[4 * q + 1] += b4.y; v[4 * q + 2] += b4.z; v[4 * q + 3] += b4.w;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < col_end) v[j] += __ldg(e.bias + col0 + j);
            }
          }
          if (e.act == 1) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = gelu_tanh_f<true>(v[j]);
          }
          if (e.resid != nullptr && row_ok) {
            const __nv_bfloat16* rr = static_cast<const __nv_bfloat16*>(e.resid) + row * e.ld_resid + col0;
            const float* g = e.gate != nullptr ? e.gate + static_cast<long long>(row / e.gate_rows) * e.ld_gate + col0
                                               : nullptr;
            if (full32) {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint4 x4 = __ldg(reinterpret_cast<const uint4*>(rr) + q);
                const uint32_t* xw = reinterpret_cast<const uint32_t*>(&x4);
                float4 g0 = make_float4(1.f, 1.f, 1.f, 1.f), g1 = g0;
                if (g != nullptr) {
                  g0 = __ldg(reinterpret_cast<const float4*>(g) + 2 * q);
                  g1 = __ldg(reinterpret_cast<const float4*>(g) + 2 * q + 1);
                }
                const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                  const float2 xf = unpack_bf16x2(xw[e2]);
                  const int j = q * 8 + 2 * e2;
                  v[j] = fmaf(gg[2 * e2], v[j], xf.x);
                  v[j + 1] = fmaf(gg[2 * e2 + 1], v[j + 1], xf.y);
                }
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < col_end) v[j] = __bfloat162float(rr[j]) + (g != nullptr ? __ldg(g + j) : 1.f) * v[j];
            }
          }
        }
        const bool f16 = col0 < p.f16_cols;   // the 32-column slice lies wholly on one side
        if (full32) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 pk;
            if (f16) {
              pk.x = pack_f16x2_sat(v[q * 8 + 0], v[q * 8 + 1]);
              pk.y = pack_f16x2_sat(v[q * 8 + 2], v[q * 8 + 3]);
              pk.z = pack_f16x2_sat(v[q * 8 + 4], v[q * 8 + 5]);
              pk.w = pack_f16x2_sat(v[q * 8 + 6], v[q * 8 + 7]);
            } else {
              pk.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
              pk.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
              pk.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
              pk.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
            }
            stg[lane * 4 + (q ^ ((lane >> 1) & 3))] = pk;
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {   // rows 8 i .. 8 i + 7 of the warp, four lanes per 64-byte segment
            const int rr = i * 8 + (lane >> 2), q = lane & 3;
            if (row0 + rr < p.M)
              reinterpret_cast<uint4*>(p.C + static_cast<size_t>(row0 + rr) * p.ldc + col0)[q] =
                  stg[rr * 4 + (q ^ ((rr >> 1) & 3))];
          }
          __syncwarp();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (col0 + j < col_end) {
              if (f16) {
                const uint32_t hh = pack_f16x2_sat(v[j], 0.f);
                reinterpret_cast<uint16_t*>(crow)[col0 + j] = static_cast<uint16_t>(hh & 0xffffu);
              } else {
                crow[col0 + j] = __float2bfloat16_rn(v[j]);
              }
            }
        }
        if (p.delta != nullptr && row_ok && col0 < p.dt_col0 + p.dt_cols && col0 + 32 > p.dt_col0) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int c = col0 + j - p.dt_col0;
            if (c >= 0 && c < p.dt_cols && col0 + j < col_end) {
              p.delta[static_cast<size_t>(row) * p.ld_delta + c] = softplus_f(__uint_as_float(r[j]) + p.dt_bias[c]);
              if (p.dt_bias2 != nullptr)
                p.delta[static_cast<size_t>(row) * p.ld_delta + p.dt_cols + c] =
                    softplus_f(__uint_as_float(r[j]) + p.dt_bias2[c]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_cta(&tempty[acc], 0));
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the leader's MMAs read this CTA's shared memory: nobody leaves before both are done
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace mate
