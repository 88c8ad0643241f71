// libmate: host side of the C ABI declared in include/mate.h.  Validates arguments, plans the caller's
// workspace, builds TMA descriptors and launches the kernels of the MATE block on the caller's stream.
// One translation unit holds every kernel, so the device status word is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/mate.h"
#include "common.cuh"
#include "gemm_bf16.cuh"
#include "simt.cuh"
#include "ssd_bf16.cuh"
#include "tesa_bf16.cuh"
#include "locality.cuh"
#include "mamba_extras.cuh"
#include "ssd_backward.cuh"
#include "dit.cuh"
#include "tesa_backward.cuh"

using namespace mate;

namespace {

thread_local int t_launches = 0;

// ------------------------------------------------------------------------------ kernel timing trace
// While a trace is on, every launch records a CUDA event before and after it on its stream.
struct Trace {
  std::mutex mu;
  std::atomic<bool> on{false};
  int cap = 0, n = 0;
  std::vector<cudaEvent_t> ev;   // 2 per record
  std::vector<int> kid;
};
Trace g_trace;
thread_local int t_trace_slot = -1;          // record opened by the last trace_begin on this thread
thread_local cudaStream_t t_trace_stream = nullptr;

void trace_begin(int kid, cudaStream_t st) {
  t_trace_slot = -1;
  if (!g_trace.on) return;
  std::lock_guard<std::mutex> lock(g_trace.mu);
  if (!g_trace.on || g_trace.n >= g_trace.cap) return;
  const int slot = g_trace.n++;
  g_trace.kid[slot] = kid;
  cudaEventRecord(g_trace.ev[2 * slot], st);
  t_trace_slot = slot;
  t_trace_stream = st;
}

void trace_end() {
  if (t_trace_slot < 0) return;
  cudaEventRecord(g_trace.ev[2 * t_trace_slot + 1], t_trace_stream);
  t_trace_slot = -1;
}

#define MATE_LAUNCH_CHECK()                         \
  do {                                              \
    ++t_launches;                                   \
    trace_end();                                    \
    if (cudaPeekAtLastError() != cudaSuccess) {     \
      (void)cudaGetLastError();                     \
      return MATE_ERR_CUDA;                         \
    }                                               \
  } while (0)

#define MATE_TRY(expr)                 \
  do {                                 \
    mate_status _s = (expr);           \
    if (_s != MATE_OK) return _s;      \
  } while (0)

constexpr int kMaxDevices = 64;
constexpr size_t kSmemLimit = 232448;  // opt-in dynamic shared memory per block on sm_100

int device_sms() {
  static int cache[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

template <typename K>
bool set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) ==
         cudaSuccess;
}

// ------------------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D matrix of 2-byte elements [rows, cols] with row stride ld (elements); box = box_rows x 64 columns,
// 128B swizzle.  The copy does not convert; the type only names the element (bf16 unless fp16 is given).
bool make_tmap(CUtensorMap* m, const void* ptr, long long rows, long long cols, long long ld, int box_rows,
               CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, type, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------------------ validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_size(const mate_config* c) { return c->dtype == MATE_BF16 ? 2 : 4; }

mate_status check_config(const mate_config* c) {
  if (c == nullptr) return MATE_ERR_ARG;
  if (c->dtype != MATE_BF16 && c->dtype != MATE_F32) return MATE_ERR_ARG;
  if (c->mamba_extras != 0 && c->mamba_extras != 1) return MATE_ERR_ARG;
  if (c->B <= 0 || c->T <= 0 || c->H <= 0 || c->W <= 0 || c->d <= 0 || c->nh <= 0 || c->P <= 0 || c->N <= 0 ||
      c->Q <= 0 || c->R < 0 || c->th <= 0 || c->tp <= 0 || c->wt <= 0 || c->wh <= 0 || c->ww <= 0)
    return MATE_ERR_SHAPE;
  if (c->T % c->wt || c->H % c->wh || c->W % c->ww) return MATE_ERR_SHAPE;
  if (c->st < 0 || c->sh < 0 || c->sw < 0 || c->st >= c->wt || c->sh >= c->wh || c->sw >= c->ww) return MATE_ERR_SHAPE;
  if (c->R % 16) return MATE_ERR_SHAPE;
  if (c->R > 0) {
    const int Tr = c->R / 16;
    if (c->T % Tr || c->H % 4 || c->W % 4) return MATE_ERR_SHAPE;
  }
  const long long n = (long long)c->T * c->H * c->W;
  if ((long long)c->B * (n + c->R) >= (1LL << 31)) return MATE_ERR_SHAPE;
  const size_t es = elem_size(c);
  if ((c->d * es) % 16 || (c->nh * c->P * es) % 16 || (c->th * c->tp * es) % 16 || (c->N * es) % 16)
    return MATE_ERR_SHAPE;
  if (c->dtype == MATE_BF16) {
    if (c->d % 64 || c->P != kSsdP || c->N != kSsdN || c->Q != kSsdQ || c->tp != 128 ||
        c->wt * c->wh * c->ww != 256 || c->nh % 8)
      return MATE_ERR_UNSUPPORTED;
  } else {
    if (c->P * c->N > 1024 || c->tp > 128) return MATE_ERR_UNSUPPORTED;
  }
  return MATE_OK;
}

// ------------------------------------------------------------------------------ workspace plans
struct Carver {
  char* base;
  size_t off = 0;
  template <typename T>
  T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

struct SsdScratch {
  __half* Gm;
  float *Sf, *Sb, *Srb;      // fp32 chunk states
  __nv_bfloat16 *Hf, *Hb;    // carried states as bf16 hi | lo pairs
  float *gl, *glb, *Gd, *tbl;
  int* crow;
};

int ceil_div(long long a, int b) { return static_cast<int>((a + b - 1) / b); }

// per_dir: also the backward scan's own decays and review-chunk states (separate backward parameters)
SsdScratch carve_ssd(Carver& cv, int B, long long n, int R, int nh, bool per_dir) {
  SsdScratch s;
  const int nRc = ceil_div(R, kSsdQ), nVc = ceil_div(n, kSsdQ);
  const size_t PN = (size_t)kSsdP * kSsdN;
  s.Gm = cv.take<__half>((size_t)B * nVc * kSsdQ * kSsdQ);
  s.Sf = cv.take<float>((size_t)B * (nRc + nVc) * nh * PN);
  s.Sb = cv.take<float>((size_t)B * nVc * nh * PN);
  s.Hf = cv.take<__nv_bfloat16>((size_t)B * nVc * nh * 2 * PN);
  s.Hb = cv.take<__nv_bfloat16>((size_t)B * nVc * nh * 2 * PN);
  s.gl = cv.take<float>((size_t)B * (nRc + nVc) * nh);
  s.glb = per_dir ? cv.take<float>((size_t)B * (nRc + nVc) * nh) : nullptr;
  s.Srb = per_dir ? cv.take<float>((size_t)B * nRc * nh * PN) : nullptr;
  s.Gd = cv.take<float>((size_t)B * nVc * kSsdQ);
  s.tbl = cv.take<float>((size_t)B * nVc * nh * 2 * kOutTbl);
  s.crow = cv.take<int>((size_t)B * nVc * kSsdQ);
  return s;
}

struct ForwardPlan {
  int NIn, NI, KO;
  int zc0;               // first gate column of the video rows' projection (mamba_extras), else -1
  void *Wi, *Wo, *Rv, *Zv, *Zr, *YO, *Ys;
  void *XBv, *XBr;       // convolved x | B | C rows (mamba_extras), same row order as Zv / Zr
  float *Dv, *Dr;
  SsdScratch ssd;
  size_t bytes;
};

ForwardPlan plan_forward(const mate_config* c, void* ws) {
  ForwardPlan p;
  Carver cv{static_cast<char*>(ws)};
  const size_t es = elem_size(c);
  const long long n = (long long)c->T * c->H * c->W;
  p.NIn = c->nh * c->P + 2 * c->N + c->nh;
  p.NI = p.NIn + 3 * c->th * c->tp;
  p.zc0 = -1;
  if (c->mamba_extras) {   // gate columns after q | k | v
    p.zc0 = p.NI;
    p.NI += c->nh * c->P;
  }
  p.KO = c->nh * c->P + c->th * c->tp;
  p.Wi = cv.take<char>((size_t)p.NI * c->d * es);
  p.Wo = cv.take<char>((size_t)c->d * p.KO * es);
  p.Rv = cv.take<char>((size_t)c->B * c->R * c->d * es);
  p.Zv = cv.take<char>((size_t)c->B * n * p.NI * es);
  p.Zr = cv.take<char>((size_t)c->B * c->R * p.NI * es);
  p.Dv = cv.take<float>((size_t)c->B * n * 2 * c->nh);      // [rows][nh forward | nh backward]
  p.Dr = cv.take<float>((size_t)c->B * c->R * 2 * c->nh);
  p.YO = cv.take<char>((size_t)c->B * n * p.KO * es);
  const size_t Cx = (size_t)c->nh * c->P + 2 * c->N;
  p.XBv = c->mamba_extras ? cv.take<char>((size_t)c->B * n * Cx * es) : nullptr;
  p.XBr = c->mamba_extras ? cv.take<char>((size_t)c->B * c->R * Cx * es) : nullptr;
  // y in scan order, for the time-fastest orders (their grid-order y rows are 1024s of rows apart)
  p.Ys = c->dtype == MATE_BF16 ? cv.take<char>((size_t)c->B * n * c->nh * c->P * es) : nullptr;
  if (c->dtype == MATE_BF16) p.ssd = carve_ssd(cv, c->B, n, c->R, c->nh, true);
  else p.ssd = SsdScratch{};
  p.bytes = cv.off + 256;
  return p;
}

size_t ssd_ws_bytes(const mate_config* c, int prefix_len, bool per_dir, float** delta, SsdScratch* s, void* ws) {
  Carver cv{static_cast<char*>(ws)};
  const long long n = (long long)c->T * c->H * c->W;
  float* d = cv.take<float>((size_t)c->B * (n + prefix_len) * (per_dir ? 2 : 1) * c->nh);
  if (delta) *delta = d;
  SsdScratch sc = c->dtype == MATE_BF16 ? carve_ssd(cv, c->B, n, prefix_len, c->nh, per_dir) : SsdScratch{};
  if (s) *s = sc;
  return cv.off + 256;
}

// ------------------------------------------------------------------------------ launchers
// Column tile of the projection GEMM.  256 wide tiles run the tensor cores best (measured against
// narrower, padding-free tiles); a ragged last tile issues narrower MMAs instead of padding.
int choose_bn(int N) { return N >= 256 ? 256 : ((N + 15) / 16) * 16; }

mate_status gemm_bf16(int kid, const void* A, int lda, long long M, int K, const void* Bw, int ldb, int N, void* C,
                      int ldc, float* delta, int ld_delta, int dt_col0, int dt_cols, const float* dt_bias,
                      cudaStream_t st, const float* dt_bias2 = nullptr, const GemmEpilogue* ep = nullptr,
                      int f16_cols = 0) {
  if (M <= 0) return MATE_OK;
  if (K % kGemmBK) return MATE_ERR_UNSUPPORTED;
  GemmParams p;
  p.M = static_cast<int>(M);
  p.N = N;
  p.K = K;
  p.bn = choose_bn(N);
  p.num_n_tiles = ceil_div(N, p.bn);
  p.C = static_cast<__nv_bfloat16*>(C);
  p.ldc = ldc;
  p.delta = delta;
  p.ld_delta = ld_delta;
  p.dt_col0 = dt_col0;
  p.dt_cols = dt_cols;
  p.dt_bias = dt_bias;
  p.dt_bias2 = dt_bias2;
  if (ep != nullptr) p.ep = *ep;
  p.f16_cols = f16_cols;
  // 256-row tiles computed by 2-CTA clusters (tcgen05 cta_group::2)
  p.num_tiles = ceil_div(M, 256) * p.num_n_tiles;
  const uint32_t psb = gemm_pair_stage_bytes(p.bn);
  p.stages = std::min<int>(8, static_cast<int>((kSmemLimit - 1024 - 256 - kGemmStageOut) / psb));
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, A, M, K, lda, 128) || !make_tmap(&tb, Bw, N, K, ldb, p.bn / 2)) return MATE_ERR_CUDA;
  const size_t smem = 1024 + (size_t)p.stages * psb + 256 + kGemmStageOut;
  if (!set_smem(gemm_bf16_pair_kernel, smem)) return MATE_ERR_CUDA;
  const int pairs = std::min(p.num_tiles, device_sms() / 2);
  trace_begin(kid, st);
  gemm_bf16_pair_kernel<<<2 * pairs, kGemmThreads, smem, st>>>(ta, tb, p);
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

mate_status gemm_f32(int kid, const float* A, int lda, long long M, int K, const float* Bw, int ldb, int N, float* C,
                     int ldc, float* delta, int ld_delta, int dt_col0, int dt_cols, const float* dt_bias,
                     cudaStream_t st, const float* dt_bias2 = nullptr, const GemmEpilogue* ep = nullptr) {
  if (M <= 0) return MATE_OK;
  dim3 grid(ceil_div(N, 64), ceil_div(M, 64));
  const GemmEpilogue e = ep != nullptr ? *ep : GemmEpilogue{};
  trace_begin(kid, st);
  gemm_f32_kernel<<<grid, 256, 0, st>>>(A, lda, Bw, ldb, C, ldc, static_cast<int>(M), N, K, delta, ld_delta, dt_col0,
                                        dt_cols, dt_bias, dt_bias2, e);
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

mate_status gather_rows(const void* src, void* dst, const mate_config* c, int order, int inverse, cudaStream_t st) {
  const long long n = (long long)c->T * c->H * c->W;
  const int vec = static_cast<int>(c->d * elem_size(c) / 16);
  const long long rows = (long long)c->B * n;
  const int blocks = static_cast<int>(std::min<long long>((rows + 7) / 8, (long long)device_sms() * 16));
  trace_begin(MATE_K_RMS_GATHER, st);
  rms_gather_rows_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), rows,
                                                 static_cast<int>(n), vec, c->T, c->H, c->W, order, inverse);
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

mate_status pool(const void* X, void* Rv, const mate_config* c, int order, cudaStream_t st) {
  if (c->R == 0) return MATE_OK;
  const int per = 16 / static_cast<int>(elem_size(c));
  const int threads = std::min(256, std::max(32, ((c->d / per) + 31) / 32 * 32));
  dim3 grid(c->R, c->B);
  trace_begin(MATE_K_REVIEW_POOL, st);
  if (c->dtype == MATE_BF16)
    review_pool_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(static_cast<const __nv_bfloat16*>(X),
                                                                static_cast<__nv_bfloat16*>(Rv), c->R, c->T, c->H,
                                                                c->W, c->d, order);
  else
    review_pool_kernel<float><<<grid, threads, 0, st>>>(static_cast<const float*>(X), static_cast<float*>(Rv), c->R,
                                                        c->T, c->H, c->W, c->d, order);
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

mate_status copy_block(const void* src, void* dst, int rows, int cols, int ld_dst, int row0, int col0, size_t es,
                       cudaStream_t st) {
  const int vcols = static_cast<int>(cols * es / 16);
  const long long total = (long long)rows * vcols;
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 4096));
  trace_begin(MATE_K_PACK_WEIGHTS, st);
  copy_block_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), rows, vcols,
                                            static_cast<int>(ld_dst * es / 16), row0, static_cast<int>(col0 * es / 16));
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

// Scan over sequences described by `rows`; y row = b*y_bstride + map(q), ldy.  bf16 or fp32 path.
mate_status run_ssd(const mate_config* c, const SeqRows& rows, const float* A_log, const float* Dp, void* y, int ldy,
                    long long y_bstride, const SsdScratch& sc, cudaStream_t st, const float* A_log_b = nullptr,
                    const float* Dp_b = nullptr) {
  const long long n = (long long)c->T * c->H * c->W;
  if (c->dtype == MATE_F32) {
    const int threads = ((c->P * c->N) + 31) / 32 * 32;
    trace_begin(MATE_K_SSD_F32, st);
    ssd_f32_kernel<<<dim3(c->nh, c->B), threads, c->P * c->N * sizeof(float), st>>>(
        rows, A_log, Dp, A_log_b, Dp_b, c->P, c->N, static_cast<float*>(y), ldy, y_bstride);
    MATE_LAUNCH_CHECK();
    return MATE_OK;
  }
  SsdBf16Params p;
  p.s = rows;
  p.B = c->B;
  p.nh = c->nh;
  p.nRc = ceil_div(rows.R, kSsdQ);
  p.nVc = ceil_div(n, kSsdQ);
  p.A_log = A_log;
  p.Dp = Dp;
  p.Gm = sc.Gm;
  p.Sf = sc.Sf;
  p.Sb = sc.Sb;
  p.gl = sc.gl;
  p.Gd = sc.Gd;
  p.Hf = sc.Hf;
  p.Hb = sc.Hb;
  p.crow = sc.crow;
  p.tbl = sc.tbl;
  p.A_log_b = A_log_b;
  p.Dp_b = Dp_b;
  p.glb = sc.glb;
  p.Srb = sc.Srb;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.ldy = ldy;
  p.y_bstride = y_bstride;
  const size_t smem_gram = 1024 + 98304 + 2048 + 64;
  const size_t smem_state = 1024 + kStSmem;
  const size_t smem_out = 1024 + kOutSmem;
  const bool xf16 = rows.x_f16 != 0;
  auto state_k = xf16 ? ssd_state_kernel<true> : ssd_state_kernel<false>;
  auto out_k = xf16 ? ssd_output_kernel<true> : ssd_output_kernel<false>;
  if (!set_smem(ssd_gram_kernel, smem_gram) || !set_smem(state_k, smem_state) || !set_smem(out_k, smem_out))
    return MATE_ERR_CUDA;
  trace_begin(MATE_K_SSD_GRAM, st);
  ssd_gram_kernel<<<dim3(p.nVc, c->B, 2), 128, smem_gram, st>>>(p);
  MATE_LAUNCH_CHECK();
  SsdStateMaps smp;
  {
    const CUtensorMapDataType xt = xf16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const long long rv = (long long)c->B * rows.v_bstride, rr = (long long)c->B * rows.r_bstride;
    smp.rows_v = static_cast<int>(rv);
    smp.rows_r = static_cast<int>(rr);
    if (!make_tmap(&smp.xv, rows.xv, rv, (long long)c->nh * c->P, rows.ldxv, 1, xt)) return MATE_ERR_CUDA;
    if (p.nRc > 0) {
      if (!make_tmap(&smp.xr, rows.xr, rr, (long long)c->nh * c->P, rows.ldxr, 1, xt)) return MATE_ERR_CUDA;
    } else {
      smp.xr = smp.xv;   // no review chunks: never read
    }
  }
  trace_begin(MATE_K_SSD_STATE, st);
  state_k<<<std::min(c->B * (p.nRc + p.nVc), device_sms()), kStThreads, smem_state, st>>>(p, smp);
  MATE_LAUNCH_CHECK();
  trace_begin(MATE_K_SSD_CARRY, st);
  ssd_carry_kernel<<<dim3(kSsdP * kSsdN / 8 / 128, c->nh, 2 * c->B), 128, 0, st>>>(p);
  MATE_LAUNCH_CHECK();
  SsdOutMaps mp;
  const long long vrows = (long long)c->B * rows.v_bstride;
  mp.rows = static_cast<int>(vrows);
  const long long srows = (long long)c->B * p.nVc * c->nh * 2 * kSsdN;   // hi | lo rows of every state
  if (!make_tmap(&mp.x, rows.xv, vrows, (long long)c->nh * c->P, rows.ldxv, 1,
                 xf16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) ||
      !make_tmap(&mp.c, rows.cv, vrows, c->N, rows.ldcv, 1) || !make_tmap(&mp.hf, sc.Hf, srows, kSsdP, kSsdP, 128) ||
      !make_tmap(&mp.hb, sc.Hb, srows, kSsdP, kSsdP, 128) ||
      !make_tmap(&mp.g, sc.Gm, (long long)c->B * p.nVc * kSsdQ, kSsdQ, kSsdQ, 128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
    return MATE_ERR_CUDA;
  const int out_groups = c->B * p.nVc * 2;
  trace_begin(MATE_K_SSD_OUTPUT, st);
  out_k<<<std::min(out_groups, device_sms()), kSsdOutThreads, smem_out, st>>>(p, mp);
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

mate_status run_tesa(const mate_config* c, const void* qkv, int ldq, int qcol, int kcol, int vcol, void* O, int ldo,
                     int ocol, int shifted, cudaStream_t st) {
  const int sft = shifted ? 1 : 0;
  if (c->dtype == MATE_F32) {
    const long long n = (long long)c->T * c->H * c->W;
    const long long warps = n * c->th;
    dim3 grid(static_cast<unsigned>((warps + 7) / 8), c->B);
    trace_begin(MATE_K_TESA_F32, st);
    tesa_f32_kernel<<<grid, 256, 0, st>>>(static_cast<const float*>(qkv), ldq, qcol, kcol, vcol,
                                          static_cast<float*>(O), ldo, ocol, c->T, c->H, c->W, c->th, c->tp, c->wt,
                                          c->wh, c->ww, c->st, c->sh, c->sw, sft);
    MATE_LAUNCH_CHECK();
    return MATE_OK;
  }
  TesaBf16Params p;
  p.qkv = static_cast<const __nv_bfloat16*>(qkv);
  p.ldq = ldq;
  p.qcol = qcol;
  p.kcol = kcol;
  p.vcol = vcol;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.ldo = ldo;
  p.ocol = ocol;
  p.B = c->B;
  p.T = c->T;
  p.H = c->H;
  p.W = c->W;
  p.th = c->th;
  p.wt = c->wt;
  p.wh = c->wh;
  p.ww = c->ww;
  p.st = sft ? c->st : 0;
  p.sh = sft ? c->sh : 0;
  p.sw = sft ? c->sw : 0;
  p.shifted = sft;
  p.scale_log2 = 1.4426950408889634f / std::sqrt(static_cast<float>(c->tp));
  const size_t smem = 1024 + kTesaSmem;
  if (!set_smem(tesa_bf16_kernel, smem)) return MATE_ERR_CUDA;
  const int nitems = (c->T / c->wt) * (c->H / c->wh) * (c->W / c->ww) * c->B * c->th;
  trace_begin(MATE_K_TESA, st);
  tesa_bf16_kernel<<<std::min(nitems, device_sms()), kTesaThreads, smem, st>>>(p);
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

// Host input and output of mate_forward_host, moved in row chunks on two copy streams so that the
// host-to-device copy overlaps the in-projection of the chunks already landed and the device-to-host copy
// overlaps the out-projection of the later chunks.  One set per device; the mutex keeps one call's
// sequence of event records and waits together.  Pipelined calls alternate between two device input
// slots; per slot the ring remembers the workspace and Out_host range of the last call that used it, the
// event after which that call no longer reads its input slot, and the event of its last output copy.
constexpr int kIoChunks = 4;
struct HostIo {
  std::mutex mu;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, in_ready[kIoChunks] = {}, out_ready[kIoChunks] = {};
  cudaEvent_t done[2] = {}, x_free[2] = {};
  const void* slot_ws[2] = {};
  uintptr_t out_lo[2] = {}, out_hi[2] = {};
  bool pending[2] = {};   // a pipelined call's output copy that no stream has been made to wait for yet
  long long calls = 0;
  bool ready = false, failed = false;
};
HostIo g_io[kMaxDevices];

HostIo* host_io() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  HostIo& io = g_io[dev];
  std::lock_guard<std::mutex> lock(io.mu);
  if (!io.ready && !io.failed) {
    bool ok = cudaStreamCreateWithFlags(&io.h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&io.d2h, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&io.start, cudaEventDisableTiming) == cudaSuccess;
    for (int k = 0; ok && k < 2; ++k)
      ok = cudaEventCreateWithFlags(&io.done[k], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&io.x_free[k], cudaEventDisableTiming) == cudaSuccess;
    for (int k = 0; ok && k < kIoChunks; ++k)
      ok = cudaEventCreateWithFlags(&io.in_ready[k], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&io.out_ready[k], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      io.failed = true;
    } else {
      io.ready = true;
    }
  }
  return io.ready ? &io : nullptr;
}

// Causal depthwise convolution + SiLU of the Cx channels [0, Cx) of the sequence rows `rows` (source
// rows rows.xv / rows.xr, strides rows.ldxv / rows.ldxr) into out_v / out_r (row stride Cx).
mate_status run_conv(const mate_config* c, const SeqRows& rows, int Cx, const float* w, const float* bias, void* out_v,
                     void* out_r, cudaStream_t st) {
  const long long L = (long long)rows.R + rows.n;
  const int nruns = ceil_div(L, kConvRun);
  const size_t es = elem_size(c);
  // 16-byte vectors when every row start and the channel count allow them
  const bool vec = (Cx * es) % 16 == 0 && (rows.ldxv * es) % 16 == 0 && (rows.ldxr * es) % 16 == 0 &&
                   aligned16(rows.xv) && aligned16(rows.xr);
  const int V = vec ? static_cast<int>(16 / es) : 1;
  const long long total = (long long)c->B * nruns * (Cx / V);
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, (long long)device_sms() * 16));
  if (total == 0) return MATE_OK;
  trace_begin(MATE_K_CONV_SILU, st);
  if (vec && (Cx * es) % 16 == 0) {
    // tiled stencil: every row load of a tile in flight at once
    const int ntp = ceil_div(L, kCvTP), ntc = ceil_div(Cx, kCvTC);
    const long long tiles = (long long)c->B * ntp * ntc;
    const size_t smem = (size_t)(kCvTP + kConvK - 1) * kCvTC * es;
    if (c->dtype == MATE_BF16) {
      if (!set_smem(conv_silu_tiled_kernel<__nv_bfloat16>, smem)) return MATE_ERR_CUDA;
      conv_silu_tiled_kernel<__nv_bfloat16><<<static_cast<unsigned>(tiles), 256, smem, st>>>(
          rows, Cx, w, bias, static_cast<__nv_bfloat16*>(out_v), static_cast<__nv_bfloat16*>(out_r), Cx, ntp, ntc);
    } else {
      if (!set_smem(conv_silu_tiled_kernel<float>, smem)) return MATE_ERR_CUDA;
      conv_silu_tiled_kernel<float><<<static_cast<unsigned>(tiles), 256, smem, st>>>(
          rows, Cx, w, bias, static_cast<float*>(out_v), static_cast<float*>(out_r), Cx, ntp, ntc);
    }
  } else if (c->dtype == MATE_BF16) {
    if (vec)
      conv_silu_kernel<__nv_bfloat16, 8><<<blocks, 256, 0, st>>>(rows, Cx, w, bias, static_cast<__nv_bfloat16*>(out_v),
                                                                static_cast<__nv_bfloat16*>(out_r), Cx, nruns, c->B);
    else
      conv_silu_kernel<__nv_bfloat16, 1><<<blocks, 256, 0, st>>>(rows, Cx, w, bias, static_cast<__nv_bfloat16*>(out_v),
                                                                static_cast<__nv_bfloat16*>(out_r), Cx, nruns, c->B);
  } else {
    if (vec)
      conv_silu_kernel<float, 4><<<blocks, 256, 0, st>>>(rows, Cx, w, bias, static_cast<float*>(out_v),
                                                         static_cast<float*>(out_r), Cx, nruns, c->B);
    else
      conv_silu_kernel<float, 1><<<blocks, 256, 0, st>>>(rows, Cx, w, bias, static_cast<float*>(out_v),
                                                         static_cast<float*>(out_r), Cx, nruns, c->B);
  }
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

// y <- gated RMSNorm(y, z) in place over rows [0, rows) (y row stride ldy, z row stride ldz, elements).
mate_status run_gate_norm(const mate_config* c, void* y, int ldy, const void* z, int ldz, const float* norm_w,
                          long long nrows, cudaStream_t st) {
  if (nrows <= 0) return MATE_OK;
  const int C = c->nh * c->P;
  const size_t es = elem_size(c);
  const bool vec = (C * es) % 16 == 0 && (ldy * es) % 16 == 0 && (ldz * es) % 16 == 0 && aligned16(y) && aligned16(z);
  const int blocks = static_cast<int>(std::min<long long>((nrows + 7) / 8, (long long)device_sms() * 16));
  trace_begin(MATE_K_GATE_NORM, st);
  if (c->dtype == MATE_BF16) {
    auto* yy = static_cast<__nv_bfloat16*>(y);
    const auto* zz = static_cast<const __nv_bfloat16*>(z);
    // rows that fit the registers: each lane holds up to 4 (or 8) 16-byte vectors of y and of z
    const bool wvec = aligned16(norm_w);   // the register kernel reads the norm weights as float4
    if (vec && wvec && C / 8 <= 32 * 4)
      gate_rmsnorm_reg_kernel<__nv_bfloat16, 4><<<blocks, 256, 0, st>>>(yy, ldy, zz, ldz, norm_w, C, nrows);
    else if (vec && wvec && C / 8 <= 32 * 8)
      gate_rmsnorm_reg_kernel<__nv_bfloat16, 8><<<blocks, 256, 0, st>>>(yy, ldy, zz, ldz, norm_w, C, nrows);
    else if (vec) gate_rmsnorm_kernel<__nv_bfloat16, 8><<<blocks, 256, 0, st>>>(yy, ldy, zz, ldz, norm_w, C, nrows);
    else gate_rmsnorm_kernel<__nv_bfloat16, 1><<<blocks, 256, 0, st>>>(yy, ldy, zz, ldz, norm_w, C, nrows);
  } else {
    auto* yy = static_cast<float*>(y);
    const auto* zz = static_cast<const float*>(z);
    if (vec) gate_rmsnorm_kernel<float, 4><<<blocks, 256, 0, st>>>(yy, ldy, zz, ldz, norm_w, C, nrows);
    else gate_rmsnorm_kernel<float, 1><<<blocks, 256, 0, st>>>(yy, ldy, zz, ldz, norm_w, C, nrows);
  }
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

// The chunked host transfers of one mate_forward_host call (null for device-buffer calls).
struct IoPlan {
  HostIo* io;
  const char* x_host;
  char* out_host;
  long long rows, chunk_rows;   // chunk c covers rows [c * chunk_rows, min(rows, (c + 1) * chunk_rows))
  size_t row_bytes;
  cudaEvent_t x_free;           // recorded on the call's stream once the device input is no longer read
};

bool cuda_ok(cudaError_t e) {
  if (e == cudaSuccess) return true;
  cudaGetLastError();
  return false;
}

// Byte offset of the packed out-projection [W_out | W_o] inside a mate_pack_weights buffer.
size_t packed_out_offset(const mate_config* c) {
  const ForwardPlan p = plan_forward(c, nullptr);
  return ((size_t)p.NI * c->d * elem_size(c) + 255) & ~size_t(255);
}

size_t packed_bytes(const mate_config* c) {
  const ForwardPlan p = plan_forward(c, nullptr);
  return packed_out_offset(c) + (size_t)c->d * p.KO * elem_size(c);
}

// [W_in; W_qkv (; W_z)] into Wi (NI x d) and [W_out | W_o] into Wo (d x KO).
mate_status pack_weights(const mate_weights* w, const mate_config* c, void* Wi, void* Wo, cudaStream_t st) {
  const ForwardPlan pl = plan_forward(c, nullptr);
  const size_t es = elem_size(c);
  const int dI = c->nh * c->P;
  MATE_TRY(copy_block(w->W_in, Wi, pl.NIn, c->d, c->d, 0, 0, es, st));
  MATE_TRY(copy_block(w->W_qkv, Wi, 3 * c->th * c->tp, c->d, c->d, pl.NIn, 0, es, st));
  if (c->mamba_extras) MATE_TRY(copy_block(w->W_z, Wi, dI, c->d, c->d, pl.zc0, 0, es, st));
  MATE_TRY(copy_block(w->W_out, Wo, c->d, dI, pl.KO, 0, 0, es, st));
  MATE_TRY(copy_block(w->W_o, Wo, c->d, c->th * c->tp, pl.KO, 0, dI, es, st));
  return MATE_OK;
}

// out_ep: optional epilogue of the out-projection (the DiT block's gated residual around the mixer).
mate_status forward_impl(const void* X, const mate_weights* w, int layer_idx, void* Out, const mate_config* c,
                         void* ws, size_t ws_bytes, cudaStream_t st, const IoPlan* iop = nullptr,
                         const GemmEpilogue* out_ep = nullptr) {
  MATE_TRY(check_config(c));
  if (X == nullptr || w == nullptr || Out == nullptr || ws == nullptr || layer_idx < 0) return MATE_ERR_ARG;
  if (w->W_in == nullptr || w->dt_bias == nullptr || w->A_log == nullptr || w->D == nullptr || w->W_out == nullptr ||
      w->W_qkv == nullptr || w->W_o == nullptr)
    return MATE_ERR_ARG;
  // separate backward-scan parameters: all three or none
  const int n_bwd = (w->dt_bias_b != nullptr) + (w->A_log_b != nullptr) + (w->D_b != nullptr);
  if (n_bwd != 0 && n_bwd != 3) return MATE_ERR_ARG;
  const bool per_dir = n_bwd == 3;
  if (!aligned16(X) || !aligned16(Out) || !aligned16(ws) || !aligned16(w->W_in) || !aligned16(w->W_out) ||
      !aligned16(w->W_qkv) || !aligned16(w->W_o))
    return MATE_ERR_ARG;
  const bool extras = c->mamba_extras == 1;
  if (extras && (w->W_z == nullptr || w->conv_w == nullptr || w->conv_b == nullptr || w->norm_w == nullptr ||
                 !aligned16(w->W_z) || !aligned16(w->conv_w)))
    return MATE_ERR_ARG;
  ForwardPlan pl = plan_forward(c, nullptr);
  if (ws_bytes < pl.bytes) return MATE_ERR_WORKSPACE;
  pl = plan_forward(c, ws);
  const int order = layer_idx % 4;
  const int shifted = layer_idx % 2;
  const size_t es = elem_size(c);
  const long long n = (long long)c->T * c->H * c->W;
  const long long Mv = (long long)c->B * n, Mr = (long long)c->B * c->R;
  const int dI = c->nh * c->P;
  const int NIn = pl.NIn, NI = pl.NI, KO = pl.KO;
  const int dt0 = dI + 2 * c->N;
  const int ldd = per_dir ? 2 * c->nh : c->nh;                     // delta rows: forward | backward
  // the scan's x columns of the projections are stored in fp16 (finer intra-chunk operand, packed fp16
  // arithmetic in the scan output kernel), except on the full-Mamba2 path whose convolution reads bf16
  const int xf16c = (c->dtype == MATE_BF16 && !extras) ? dI : 0;
  const float* dtb2 = per_dir ? w->dt_bias_b : nullptr;

  // packed weights: Wi = [W_in; W_qkv (; W_z)] (NI x d), Wo = [W_out | W_o] (d x KO), from the caller's
  // mate_pack_weights buffer when given, else packed into the workspace on every call
  if (w->packed != nullptr) {
    if (!aligned16(w->packed)) return MATE_ERR_ARG;
    pl.Wi = const_cast<void*>(w->packed);
    pl.Wo = static_cast<char*>(pl.Wi) + packed_out_offset(c);
  } else {
    MATE_TRY(pack_weights(w, c, pl.Wi, pl.Wo, st));
  }
  // review tokens, then the projections of the video rows (grid order) and of the review rows
  if (c->dtype == MATE_BF16 && iop != nullptr) {
    // host input: project each row chunk as soon as it has landed; the review pool needs all of X
    for (int k = 0; k < kIoChunks; ++k) {
      const long long r0 = k * iop->chunk_rows, r1 = std::min(iop->rows, r0 + iop->chunk_rows);
      if (!cuda_ok(cudaStreamWaitEvent(st, iop->io->in_ready[k], 0))) return MATE_ERR_CUDA;
      if (r1 <= r0) continue;
      MATE_TRY(gemm_bf16(MATE_K_IN_PROJ, static_cast<const char*>(X) + r0 * c->d * es, c->d, r1 - r0, c->d, pl.Wi,
                         c->d, NI, static_cast<char*>(pl.Zv) + r0 * NI * es, NI, pl.Dv + r0 * ldd, ldd, dt0,
                         c->nh, w->dt_bias, st, dtb2, nullptr, xf16c));
    }
    MATE_TRY(pool(X, pl.Rv, c, order, st));
    if (!cuda_ok(cudaEventRecord(iop->x_free, st))) return MATE_ERR_CUDA;
    MATE_TRY(gemm_bf16(MATE_K_IN_PROJ_REVIEW, pl.Rv, c->d, Mr, c->d, pl.Wi, c->d, NIn, pl.Zr, NI, pl.Dr, ldd, dt0,
                       c->nh, w->dt_bias, st, dtb2, nullptr, xf16c));
  } else if (c->dtype == MATE_BF16) {
    MATE_TRY(pool(X, pl.Rv, c, order, st));
    MATE_TRY(gemm_bf16(MATE_K_IN_PROJ, X, c->d, Mv, c->d, pl.Wi, c->d, NI, pl.Zv, NI, pl.Dv, ldd, dt0, c->nh,
                       w->dt_bias, st, dtb2, nullptr, xf16c));
    MATE_TRY(gemm_bf16(MATE_K_IN_PROJ_REVIEW, pl.Rv, c->d, Mr, c->d, pl.Wi, c->d, NIn, pl.Zr, NI, pl.Dr, ldd, dt0,
                       c->nh, w->dt_bias, st, dtb2, nullptr, xf16c));
  } else {
    MATE_TRY(pool(X, pl.Rv, c, order, st));
    MATE_TRY(gemm_f32(MATE_K_IN_PROJ, static_cast<const float*>(X), c->d, Mv, c->d, static_cast<const float*>(pl.Wi), c->d, NI,
                      static_cast<float*>(pl.Zv), NI, pl.Dv, ldd, dt0, c->nh, w->dt_bias, st, dtb2));
    MATE_TRY(gemm_f32(MATE_K_IN_PROJ_REVIEW, static_cast<const float*>(pl.Rv), c->d, Mr, c->d, static_cast<const float*>(pl.Wi), c->d, NIn,
                      static_cast<float*>(pl.Zr), NI, pl.Dr, ldd, dt0, c->nh, w->dt_bias, st, dtb2));
  }
  // MA: scan over [review rows; video rows in scan order], y written at grid-order rows of YO[:, :dI]
  SeqRows rows;
  const char* zv = static_cast<const char*>(pl.Zv);
  const char* zr = static_cast<const char*>(pl.Zr);
  rows.xv = zv;
  rows.bv = zv + (size_t)dI * es;
  rows.cv = zv + (size_t)(dI + c->N) * es;
  rows.dv = pl.Dv;
  rows.xr = zr;
  rows.br = zr + (size_t)dI * es;
  rows.cr = zr + (size_t)(dI + c->N) * es;
  rows.dr = pl.Dr;
  rows.ldxv = rows.ldbv = rows.ldcv = NI;
  rows.ldxr = rows.ldbr = rows.ldcr = NI;
  rows.lddv = rows.lddr = ldd;
  rows.db_off = per_dir ? c->nh : 0;
  rows.v_bstride = n;
  rows.v_off = 0;
  rows.r_bstride = c->R;
  rows.r_off = 0;
  rows.n = static_cast<int>(n);
  rows.R = c->R;
  rows.T = c->T;
  rows.H = c->H;
  rows.W = c->W;
  rows.order = order;
  if (extras) {
    // x | B | C through the causal convolution + SiLU, along [review rows; video rows in scan order];
    // the scan then reads the convolved rows (same row order, row stride Cx)
    const int Cx = dI + 2 * c->N;
    MATE_TRY(run_conv(c, rows, Cx, w->conv_w, w->conv_b, pl.XBv, pl.XBr, st));
    const char* xbv = static_cast<const char*>(pl.XBv);
    const char* xbr = static_cast<const char*>(pl.XBr);
    rows.xv = xbv;
    rows.bv = xbv + (size_t)dI * es;
    rows.cv = xbv + (size_t)(dI + c->N) * es;
    rows.xr = xbr;
    rows.br = xbr + (size_t)dI * es;
    rows.cr = xbr + (size_t)(dI + c->N) * es;
    rows.ldxv = rows.ldbv = rows.ldcv = Cx;
    rows.ldxr = rows.ldbr = rows.ldcr = Cx;
  }
  // Orders 2 and 3 run time fastest: grid-order rows of one chunk lie in 256 different time planes, and
  // writing each head's 128-byte y piece there costs more than writing y in scan order and moving whole
  // rows back to grid order afterwards (measured on the B200).
  const bool y_in_scan_order = c->dtype == MATE_BF16 && order >= 2;
  rows.y_order = y_in_scan_order ? -1 : order;
  rows.x_f16 = xf16c > 0 ? 1 : 0;
  if (y_in_scan_order) {
    MATE_TRY(run_ssd(c, rows, w->A_log, w->D, pl.Ys, dI, n, pl.ssd, st, w->A_log_b, w->D_b));
    const int vec = static_cast<int>(dI * es / 16);
    const long long total = (long long)c->B * n;
    const int blocks = static_cast<int>(std::min<long long>((total + 7) / 8, (long long)device_sms() * 16));
    trace_begin(MATE_K_Y_TO_GRID, st);
    scan_rows_to_grid_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint4*>(pl.Ys), vec,
                                                    static_cast<uint4*>(pl.YO), static_cast<long long>(KO * es / 16),
                                                    vec, total, static_cast<int>(n), c->T, c->H, c->W, order);
    MATE_LAUNCH_CHECK();
  } else {
    MATE_TRY(run_ssd(c, rows, w->A_log, w->D, pl.YO, KO, n, pl.ssd, st, w->A_log_b, w->D_b));
  }
  // gate and gated RMSNorm of y in place (grid-order rows of YO[:, :dI]), before the out-projection
  if (extras) MATE_TRY(run_gate_norm(c, pl.YO, KO, static_cast<const char*>(pl.Zv) + (size_t)pl.zc0 * es, NI, w->norm_w,
                                     Mv, st));
  // TE: window attention on the q | k | v columns of Zv, output into YO[:, dI:]
  const int qc = NIn, ac = c->th * c->tp;
  MATE_TRY(run_tesa(c, pl.Zv, NI, qc, qc + ac, qc + 2 * ac, pl.YO, KO, dI, shifted, st));
  // Out = [y | O] [W_out | W_o]^T = MA + TE
  if (c->dtype == MATE_BF16 && iop != nullptr) {
    // host output: each row chunk goes back to the host while the later chunks are projected
    for (int k = 0; k < kIoChunks; ++k) {
      const long long r0 = k * iop->chunk_rows, r1 = std::min(iop->rows, r0 + iop->chunk_rows);
      if (r1 > r0)
        MATE_TRY(gemm_bf16(MATE_K_OUT_PROJ, static_cast<const char*>(pl.YO) + r0 * KO * es, KO, r1 - r0, KO, pl.Wo,
                           KO, c->d, static_cast<char*>(Out) + r0 * c->d * es, c->d, nullptr, 0, 0, 0, nullptr, st));
      if (!cuda_ok(cudaEventRecord(iop->io->out_ready[k], st)) ||
          !cuda_ok(cudaStreamWaitEvent(iop->io->d2h, iop->io->out_ready[k], 0)))
        return MATE_ERR_CUDA;
      if (r1 > r0 && !cuda_ok(cudaMemcpyAsync(iop->out_host + r0 * iop->row_bytes,
                                              static_cast<const char*>(Out) + r0 * iop->row_bytes,
                                              (r1 - r0) * iop->row_bytes, cudaMemcpyDeviceToHost, iop->io->d2h)))
        return MATE_ERR_CUDA;
    }
  } else if (c->dtype == MATE_BF16)
    MATE_TRY(gemm_bf16(MATE_K_OUT_PROJ, pl.YO, KO, Mv, KO, pl.Wo, KO, c->d, Out, c->d, nullptr, 0, 0, 0, nullptr, st,
                       nullptr, out_ep));
  else
    MATE_TRY(gemm_f32(MATE_K_OUT_PROJ, static_cast<const float*>(pl.YO), KO, Mv, KO, static_cast<const float*>(pl.Wo), KO, c->d,
                      static_cast<float*>(Out), c->d, nullptr, 0, 0, 0, nullptr, st, nullptr, out_ep));
  return MATE_OK;
}

}  // namespace

extern "C" {

const char* mate_status_str(mate_status s) {
  switch (s) {
    case MATE_OK: return "ok";
    case MATE_ERR_ARG: return "invalid argument";
    case MATE_ERR_SHAPE: return "inconsistent shape";
    case MATE_ERR_WORKSPACE: return "workspace too small";
    case MATE_ERR_CUDA: return "CUDA error";
    case MATE_ERR_TIMEOUT: return "device wait timed out";
    case MATE_ERR_UNSUPPORTED: return "shape not supported by the tensor-core kernels";
    case MATE_ERR_TOO_LARGE: return "problem needs more scratch than the fixed device buffer holds";
  }
  return "unknown status";
}

mate_status mate_check_config(const mate_config* cfg) { return check_config(cfg); }

size_t mate_workspace_bytes(const mate_config* cfg) {
  if (check_config(cfg) != MATE_OK) return 0;
  return plan_forward(cfg, nullptr).bytes;
}

size_t mate_ssd_workspace_bytes(const mate_config* cfg, int prefix_len) {
  if (check_config(cfg) != MATE_OK || prefix_len < 0) return 0;
  return ssd_ws_bytes(cfg, prefix_len, false, nullptr, nullptr, nullptr);
}

size_t mate_ssd_pd_workspace_bytes(const mate_config* cfg, int prefix_len) {
  if (check_config(cfg) != MATE_OK || prefix_len < 0) return 0;
  return ssd_ws_bytes(cfg, prefix_len, true, nullptr, nullptr, nullptr);
}

size_t mate_forward_host_workspace_bytes(const mate_config* cfg) {
  if (check_config(cfg) != MATE_OK) return 0;
  const size_t xb = (size_t)cfg->B * cfg->T * cfg->H * cfg->W * cfg->d * elem_size(cfg);
  // the block's workspace, two device input slots and two device output slots (pipelined calls alternate)
  return mate_workspace_bytes(cfg) + 4 * ((xb + 255) & ~size_t(255));
}

mate_status rms_permute(const void* X, void* Xp, int order, const mate_config* cfg, mate_stream_t stream) {
  MATE_TRY(check_config(cfg));
  if (X == nullptr || Xp == nullptr || order < 0 || order > 3 || !aligned16(X) || !aligned16(Xp)) return MATE_ERR_ARG;
  t_launches = 0;
  return gather_rows(X, Xp, cfg, order, 0, reinterpret_cast<cudaStream_t>(stream));
}

mate_status rms_unpermute(const void* Xp, void* X, int order, const mate_config* cfg, mate_stream_t stream) {
  MATE_TRY(check_config(cfg));
  if (X == nullptr || Xp == nullptr || order < 0 || order > 3 || !aligned16(X) || !aligned16(Xp)) return MATE_ERR_ARG;
  t_launches = 0;
  return gather_rows(Xp, X, cfg, order, 1, reinterpret_cast<cudaStream_t>(stream));
}

mate_status review_pool(const void* X, void* Rv, int order, const mate_config* cfg, mate_stream_t stream) {
  MATE_TRY(check_config(cfg));
  if (X == nullptr || (Rv == nullptr && cfg->R > 0) || order < 0 || order > 3 || !aligned16(X) || !aligned16(Rv))
    return MATE_ERR_ARG;
  t_launches = 0;
  return pool(X, Rv, cfg, order, reinterpret_cast<cudaStream_t>(stream));
}

mate_status scan_impl(const void* x, const void* Bm, const void* Cm, const float* dt, const float* dt_bias,
                      const float* A_log, const float* D, const float* dt_bias_b, const float* A_log_b,
                      const float* D_b, int prefix_len, void* y, const mate_config* cfg, void* ws, size_t ws_bytes,
                      mate_stream_t stream) {
  MATE_TRY(check_config(cfg));
  if (x == nullptr || Bm == nullptr || Cm == nullptr || dt == nullptr || dt_bias == nullptr || A_log == nullptr ||
      D == nullptr || y == nullptr || ws == nullptr || prefix_len < 0)
    return MATE_ERR_ARG;
  if (!aligned16(x) || !aligned16(Bm) || !aligned16(Cm) || !aligned16(y) || !aligned16(ws)) return MATE_ERR_ARG;
  const int n_bwd = (dt_bias_b != nullptr) + (A_log_b != nullptr) + (D_b != nullptr);
  if (n_bwd != 0 && n_bwd != 3) return MATE_ERR_ARG;
  const bool per_dir = n_bwd == 3;
  if (ws_bytes < ssd_ws_bytes(cfg, prefix_len, per_dir, nullptr, nullptr, nullptr)) return MATE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_launches = 0;
  float* delta = nullptr;
  SsdScratch sc;
  ssd_ws_bytes(cfg, prefix_len, per_dir, &delta, &sc, ws);
  const long long n = (long long)cfg->T * cfg->H * cfg->W;
  const long long L = n + prefix_len;
  const long long total = (long long)cfg->B * L * cfg->nh;
  trace_begin(MATE_K_SOFTPLUS, st);
  softplus_kernel<<<static_cast<int>(std::min<long long>((total + 255) / 256, 4096)), 256, 0, st>>>(
      dt, dt_bias, per_dir ? dt_bias_b : nullptr, delta, total, cfg->nh);
  MATE_LAUNCH_CHECK();
  SeqRows rows;
  rows.xv = rows.xr = x;
  rows.bv = rows.br = Bm;
  rows.cv = rows.cr = Cm;
  rows.dv = rows.dr = delta;
  rows.ldxv = rows.ldxr = cfg->nh * cfg->P;
  rows.ldbv = rows.ldbr = rows.ldcv = rows.ldcr = cfg->N;
  rows.lddv = rows.lddr = per_dir ? 2 * cfg->nh : cfg->nh;
  rows.db_off = per_dir ? cfg->nh : 0;
  rows.v_bstride = L;
  rows.v_off = prefix_len;
  rows.r_bstride = L;
  rows.r_off = 0;
  rows.n = static_cast<int>(n);
  rows.R = prefix_len;
  rows.T = cfg->T;
  rows.H = cfg->H;
  rows.W = cfg->W;
  rows.order = -1;
  rows.y_order = -1;
  return run_ssd(cfg, rows, A_log, D, y, cfg->nh * cfg->P, n, sc, st, per_dir ? A_log_b : nullptr,
                 per_dir ? D_b : nullptr);
}

mate_status ssd_scan_bidir(const void* x, const void* Bm, const void* Cm, const float* dt, const float* dt_bias,
                           const float* A_log, const float* D, int prefix_len, void* y, const mate_config* cfg,
                           void* ws, size_t ws_bytes, mate_stream_t stream) {
  return scan_impl(x, Bm, Cm, dt, dt_bias, A_log, D, nullptr, nullptr, nullptr, prefix_len, y, cfg, ws, ws_bytes,
                   stream);
}

mate_status ssd_scan_bidir_pd(const void* x, const void* Bm, const void* Cm, const float* dt, const float* dt_bias,
                              const float* A_log, const float* D, const float* dt_bias_b, const float* A_log_b,
                              const float* D_b, int prefix_len, void* y, const mate_config* cfg, void* ws,
                              size_t ws_bytes, mate_stream_t stream) {
  if (dt_bias_b == nullptr || A_log_b == nullptr || D_b == nullptr) return MATE_ERR_ARG;
  return scan_impl(x, Bm, Cm, dt, dt_bias, A_log, D, dt_bias_b, A_log_b, D_b, prefix_len, y, cfg, ws, ws_bytes,
                   stream);
}

size_t mate_ssd_backward_workspace_bytes(const mate_config* cfg, int prefix_len) {
  if (check_config(cfg) != MATE_OK || prefix_len < 0) return 0;
  const long long L = (long long)cfg->T * cfg->H * cfg->W + prefix_len;
  return (size_t)cfg->B * cfg->nh * L * cfg->P * cfg->N * sizeof(float) + 256;
}

mate_status ssd_scan_bidir_backward(const void* x, const void* Bm, const void* Cm, const float* dt,
                                    const float* dt_bias, const float* A_log, const float* D, int prefix_len,
                                    const void* dy, void* dx, void* dB, void* dC, float* ddt, float* ddt_bias,
                                    float* dA_log, float* dD, const mate_config* cfg, void* ws, size_t ws_bytes,
                                    mate_stream_t stream) {
  MATE_TRY(check_config(cfg));
  if (x == nullptr || Bm == nullptr || Cm == nullptr || dt == nullptr || dt_bias == nullptr || A_log == nullptr ||
      D == nullptr || dy == nullptr || dx == nullptr || dB == nullptr || dC == nullptr || ddt == nullptr ||
      ddt_bias == nullptr || dA_log == nullptr || dD == nullptr || ws == nullptr || prefix_len < 0)
    return MATE_ERR_ARG;
  if (cfg->dtype != MATE_F32) return MATE_ERR_UNSUPPORTED;
  if (ws_bytes < mate_ssd_backward_workspace_bytes(cfg, prefix_len)) return MATE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_launches = 0;
  const long long n = (long long)cfg->T * cfg->H * cfg->W;
  const long long L = n + prefix_len;
  if (!cuda_ok(cudaMemsetAsync(dB, 0, (size_t)cfg->B * L * cfg->N * sizeof(float), st)) ||
      !cuda_ok(cudaMemsetAsync(dC, 0, (size_t)cfg->B * L * cfg->N * sizeof(float), st)) ||
      !cuda_ok(cudaMemsetAsync(ddt_bias, 0, (size_t)cfg->nh * sizeof(float), st)) ||
      !cuda_ok(cudaMemsetAsync(dA_log, 0, (size_t)cfg->nh * sizeof(float), st)) ||
      !cuda_ok(cudaMemsetAsync(dD, 0, (size_t)cfg->nh * sizeof(float), st)))
    return MATE_ERR_CUDA;
  SeqRows rows;
  rows.xv = rows.xr = x;
  rows.bv = rows.br = Bm;
  rows.cv = rows.cr = Cm;
  rows.dv = rows.dr = nullptr;
  rows.ldxv = rows.ldxr = cfg->nh * cfg->P;
  rows.ldbv = rows.ldbr = rows.ldcv = rows.ldcr = cfg->N;
  rows.lddv = rows.lddr = cfg->nh;
  rows.db_off = 0;
  rows.v_bstride = L;
  rows.v_off = prefix_len;
  rows.r_bstride = L;
  rows.r_off = 0;
  rows.n = static_cast<int>(n);
  rows.R = prefix_len;
  rows.T = cfg->T;
  rows.H = cfg->H;
  rows.W = cfg->W;
  rows.order = -1;
  rows.y_order = -1;
  const int PN = cfg->P * cfg->N;
  const int threads = (PN + 31) / 32 * 32;
  const size_t smem = (size_t)(4 * PN + 3 * cfg->P) * sizeof(float);
  trace_begin(MATE_K_SSD_BACKWARD, st);
  ssd_backward_f32_kernel<<<dim3(cfg->nh, cfg->B), threads, smem, st>>>(
      rows, dt, cfg->nh, dt_bias, A_log, D, cfg->P, cfg->N, static_cast<const float*>(dy), static_cast<float*>(dx),
      static_cast<float*>(dB), static_cast<float*>(dC), ddt, ddt_bias, dA_log, dD, static_cast<float*>(ws));
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

// Fixed scratch behind ssd_scan_bidir_noalloc.  In host code this name is only a stand-in for the
// device symbol; its device address comes from cudaGetSymbolAddress, once per device and CUDA context.
static __device__ __align__(256) unsigned char g_ssd_noalloc_scratch[MATE_SSD_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kNoallocMaxDevices = 128;
std::mutex g_noalloc_mutex;
// Device address of the scratch by device ordinal, with the CUDA context it was looked up in: the array
// lives in the library's device code loaded into that context, so after cudaDeviceReset (a new context)
// the address is looked up again.
struct NoallocAddr {
  CUcontext ctx;
  void* addr;
};
NoallocAddr g_noalloc_addr[kNoallocMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}
}  // namespace

mate_status ssd_scan_bidir_noalloc(const void* x, const void* Bm, const void* Cm, const float* dt,
                                   const float* dt_bias, const float* A_log, const float* D, int prefix_len, void* y,
                                   const mate_config* cfg, mate_stream_t stream) {
  MATE_TRY(check_config(cfg));
  if (prefix_len < 0) return MATE_ERR_ARG;
  if (ssd_ws_bytes(cfg, prefix_len, false, nullptr, nullptr, nullptr) > MATE_SSD_NOALLOC_SCRATCH_BYTES)
    return MATE_ERR_TOO_LARGE;
  if (x == nullptr || Bm == nullptr || Cm == nullptr || dt == nullptr || dt_bias == nullptr || A_log == nullptr ||
      D == nullptr || y == nullptr)
    return MATE_ERR_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) {
    cudaGetLastError();
    return MATE_ERR_CUDA;
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    // cudaGetSymbolAddress also makes the context current and loads the device code if needed, so the
    // context is read after it on the first call
    const CUcontext ctx = current_context();
    NoallocAddr& na = g_noalloc_addr[dev];
    if (na.addr == nullptr || ctx == nullptr || na.ctx != ctx) {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_ssd_noalloc_scratch) != cudaSuccess || addr == nullptr) {
        cudaGetLastError();
        return MATE_ERR_CUDA;
      }
      na.addr = addr;
      na.ctx = current_context();
    }
    scratch = na.addr;
  }
  return ssd_scan_bidir(x, Bm, Cm, dt, dt_bias, A_log, D, prefix_len, y, cfg, scratch, MATE_SSD_NOALLOC_SCRATCH_BYTES,
                        stream);
}

mate_status tesa_forward(const void* qkv, void* O, int shifted, const mate_config* cfg, mate_stream_t stream) {
  MATE_TRY(check_config(cfg));
  if (qkv == nullptr || O == nullptr || !aligned16(qkv) || !aligned16(O)) return MATE_ERR_ARG;
  t_launches = 0;
  const int a = cfg->th * cfg->tp;
  return run_tesa(cfg, qkv, 3 * a, 0, a, 2 * a, O, a, 0, shifted, reinterpret_cast<cudaStream_t>(stream));
}

mate_status mate_scan_locality(int T, int H, int W, int map, unsigned long long* out, mate_stream_t stream) {
  if (out == nullptr || T <= 0 || H <= 0 || W <= 0 || map < 0 || map > 6 || (reinterpret_cast<uintptr_t>(out) & 7))
    return MATE_ERR_ARG;
  if (static_cast<long long>(T) * H * W >= (1LL << 31)) return MATE_ERR_SHAPE;
  int bits = 1;
  if (map == 5) {
    if (H != W || (H & (H - 1)) != 0 || T % H != 0) return MATE_ERR_UNSUPPORTED;
    while ((1 << bits) < H) ++bits;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_launches = 0;
  if (cudaMemsetAsync(out, 0, 3 * sizeof(unsigned long long), st) != cudaSuccess) {
    cudaGetLastError();
    return MATE_ERR_CUDA;
  }
  const long long n = static_cast<long long>(T) * H * W;
  const int blocks = static_cast<int>(std::min<long long>((n + 255) / 256, (long long)device_sms() * 8));
  trace_begin(MATE_K_SCAN_LOCALITY, st);
  scan_locality_kernel<<<blocks, 256, 0, st>>>(T, H, W, map, bits, out);
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

mate_status mate_project_bf16(const void* A, int lda, long long M, int K, const void* Wt, int ldw, int N, void* C,
                              int ldc, mate_stream_t stream) {
  if (A == nullptr || Wt == nullptr || C == nullptr || M < 0 || K <= 0 || N <= 0) return MATE_ERR_ARG;
  if (!aligned16(A) || !aligned16(Wt) || !aligned16(C) || lda % 8 || ldw % 8 || ldc % 8 || lda < K || ldw < K ||
      ldc < N || M >= (1LL << 31))
    return MATE_ERR_ARG;
  if (K % kGemmBK) return MATE_ERR_UNSUPPORTED;
  t_launches = 0;
  return gemm_bf16(MATE_K_PROJECT, A, lda, M, K, Wt, ldw, N, C, ldc, nullptr, 0, 0, 0, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

mate_status mate_forward(const void* X, const mate_weights* w, int layer_idx, void* Out, const mate_config* cfg,
                         void* ws, size_t ws_bytes, mate_stream_t stream) {
  t_launches = 0;
  return forward_impl(X, w, layer_idx, Out, cfg, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {
bool ranges_overlap(uintptr_t a0, uintptr_t a1, uintptr_t b0, uintptr_t b1) { return a0 < b1 && b0 < a1; }

mate_status forward_host_impl(const void* X_host, const mate_weights* w, int layer_idx, void* Out_host,
                              const mate_config* cfg, void* ws, size_t ws_bytes, cudaStream_t st, bool pipelined) {
  MATE_TRY(check_config(cfg));
  if (X_host == nullptr || Out_host == nullptr || ws == nullptr) return MATE_ERR_ARG;
  if (ws_bytes < mate_forward_host_workspace_bytes(cfg)) return MATE_ERR_WORKSPACE;
  const size_t fw = mate_workspace_bytes(cfg);
  const size_t xb = (size_t)cfg->B * cfg->T * cfg->H * cfg->W * cfg->d * elem_size(cfg);
  const size_t xb_al = (xb + 255) & ~size_t(255);
  char* xslot0 = static_cast<char*>(ws) + ((fw + 255) & ~size_t(255));
  t_launches = 0;
  HostIo* io = cfg->dtype == MATE_BF16 ? host_io() : nullptr;
  if (io == nullptr) {   // one copy each way on `stream`
    char* odev = xslot0 + 2 * xb_al;
    if (cudaMemcpyAsync(xslot0, X_host, xb, cudaMemcpyHostToDevice, st) != cudaSuccess) return MATE_ERR_CUDA;
    MATE_TRY(forward_impl(xslot0, w, layer_idx, odev, cfg, ws, fw, st));
    if (cudaMemcpyAsync(Out_host, odev, xb, cudaMemcpyDeviceToHost, st) != cudaSuccess) return MATE_ERR_CUDA;
    return MATE_OK;
  }
  std::lock_guard<std::mutex> lock(io->mu);
  const int slot = pipelined ? static_cast<int>(io->calls & 1) : 0;
  char* xdev = xslot0 + slot * xb_al;
  char* odev = xslot0 + (2 + slot) * xb_al;
  if (!pipelined) {   // no earlier pipelined output copy may still be running when this call starts
    for (int j = 0; j < 2; ++j)
      if (io->pending[j]) {
        if (!cuda_ok(cudaStreamWaitEvent(st, io->done[j], 0))) return MATE_ERR_CUDA;
        io->pending[j] = false;
      }
  }
  IoPlan iop;
  iop.io = io;
  iop.x_host = static_cast<const char*>(X_host);
  iop.out_host = static_cast<char*>(Out_host);
  iop.rows = (long long)cfg->B * cfg->T * cfg->H * cfg->W;
  iop.row_bytes = (size_t)cfg->d * elem_size(cfg);
  iop.chunk_rows = ((iop.rows + kIoChunks - 1) / kIoChunks + 255) / 256 * 256;
  iop.x_free = io->x_free[slot];
  const uintptr_t x0 = reinterpret_cast<uintptr_t>(X_host), o0 = reinterpret_cast<uintptr_t>(Out_host);
  if (!pipelined || io->slot_ws[slot] != ws) {
    // the copies start after all earlier work on `stream` (the workspace may still be in use)
    if (!cuda_ok(cudaEventRecord(io->start, st)) || !cuda_ok(cudaStreamWaitEvent(io->h2d, io->start, 0)) ||
        !cuda_ok(cudaStreamWaitEvent(io->d2h, io->start, 0)))
      return MATE_ERR_CUDA;
  } else {
    // the input copy waits only until the call that last used this input slot has read it, and for the
    // output copies of earlier calls whose Out_host overlaps X_host; everything else of the previous call
    // (its output copies included) may still run
    if (!cuda_ok(cudaStreamWaitEvent(io->h2d, io->x_free[slot], 0))) return MATE_ERR_CUDA;
    for (int j = 0; j < 2; ++j)
      if (ranges_overlap(x0, x0 + xb, io->out_lo[j], io->out_hi[j]) &&
          !cuda_ok(cudaStreamWaitEvent(io->h2d, io->done[j], 0)))
        return MATE_ERR_CUDA;
  }
  for (int k = 0; k < kIoChunks; ++k) {
    const long long r0 = k * iop.chunk_rows, r1 = std::min(iop.rows, r0 + iop.chunk_rows);
    if (r1 > r0 && !cuda_ok(cudaMemcpyAsync(xdev + r0 * iop.row_bytes, iop.x_host + r0 * iop.row_bytes,
                                            (r1 - r0) * iop.row_bytes, cudaMemcpyHostToDevice, io->h2d)))
      return MATE_ERR_CUDA;
    if (!cuda_ok(cudaEventRecord(io->in_ready[k], io->h2d))) return MATE_ERR_CUDA;
  }
  MATE_TRY(forward_impl(xdev, w, layer_idx, odev, cfg, ws, fw, st, &iop));
  if (!cuda_ok(cudaEventRecord(io->done[slot], io->d2h))) return MATE_ERR_CUDA;
  if (!pipelined) {
    // the call ends on `stream` only when the last chunk has reached the host
    if (!cuda_ok(cudaStreamWaitEvent(st, io->done[slot], 0))) return MATE_ERR_CUDA;
  } else {
    // this call's output copy runs on beside the next call's work; the stream waits here for the previous
    // call's output copy (whose device output slot the next call overwrites)
    const int prev = slot ^ 1;
    if (io->pending[prev]) {
      if (!cuda_ok(cudaStreamWaitEvent(st, io->done[prev], 0))) return MATE_ERR_CUDA;
      io->pending[prev] = false;
    }
    io->pending[slot] = true;
  }
  io->slot_ws[slot] = ws;
  io->out_lo[slot] = o0;
  io->out_hi[slot] = o0 + xb;
  ++io->calls;
  return MATE_OK;
}
}  // namespace

extern "C" {

mate_status mate_forward_host(const void* X_host, const mate_weights* w, int layer_idx, void* Out_host,
                              const mate_config* cfg, void* ws, size_t ws_bytes, mate_stream_t stream) {
  return forward_host_impl(X_host, w, layer_idx, Out_host, cfg, ws, ws_bytes,
                           reinterpret_cast<cudaStream_t>(stream), false);
}

mate_status mate_forward_host_pipelined(const void* X_host, const mate_weights* w, int layer_idx, void* Out_host,
                                        const mate_config* cfg, void* ws, size_t ws_bytes, mate_stream_t stream) {
  return forward_host_impl(X_host, w, layer_idx, Out_host, cfg, ws, ws_bytes,
                           reinterpret_cast<cudaStream_t>(stream), true);
}

mate_status mate_forward_host_flush(mate_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return MATE_ERR_CUDA;
  }
  HostIo& io = g_io[dev];
  std::lock_guard<std::mutex> lock(io.mu);
  if (!io.ready) return MATE_OK;
  for (int j = 0; j < 2; ++j)
    if (io.pending[j]) {
      if (!cuda_ok(cudaStreamWaitEvent(st, io.done[j], 0))) return MATE_ERR_CUDA;
      io.pending[j] = false;
    }
  return MATE_OK;
}

size_t mate_packed_weights_bytes(const mate_config* cfg) {
  if (check_config(cfg) != MATE_OK) return 0;
  return packed_bytes(cfg);
}

mate_status mate_pack_weights(const mate_weights* w, const mate_config* cfg, void* packed, size_t packed_bytes_,
                              mate_stream_t stream) {
  MATE_TRY(check_config(cfg));
  if (w == nullptr || packed == nullptr || !aligned16(packed) || w->W_in == nullptr || w->W_out == nullptr ||
      w->W_qkv == nullptr || w->W_o == nullptr || !aligned16(w->W_in) || !aligned16(w->W_out) ||
      !aligned16(w->W_qkv) || !aligned16(w->W_o))
    return MATE_ERR_ARG;
  if (cfg->mamba_extras && (w->W_z == nullptr || !aligned16(w->W_z))) return MATE_ERR_ARG;
  if (packed_bytes_ < packed_bytes(cfg)) return MATE_ERR_WORKSPACE;
  t_launches = 0;
  return pack_weights(w, cfg, packed, static_cast<char*>(packed) + packed_out_offset(cfg),
                      reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {
struct DitPlan {
  float* mod;   // [B][6][d] modulation
  void *h, *X1, *Z;
  void* mate_ws;
  size_t mate_bytes, bytes;
};

DitPlan plan_dit(const mate_config* c, void* ws) {
  DitPlan p;
  Carver cv{static_cast<char*>(ws)};
  const size_t es = elem_size(c);
  const size_t rows = (size_t)c->B * c->T * c->H * c->W;
  p.mod = cv.take<float>((size_t)c->B * 6 * c->d);
  p.h = cv.take<char>(rows * c->d * es);
  p.X1 = cv.take<char>(rows * c->d * es);
  p.Z = cv.take<char>(rows * 4 * c->d * es);
  p.mate_bytes = plan_forward(c, nullptr).bytes;
  p.mate_ws = cv.take<char>(p.mate_bytes);
  p.bytes = cv.off + 256;
  return p;
}

mate_status ln_modulate(const mate_config* c, const void* x, void* h, const float* shift, const float* scale,
                        cudaStream_t st) {
  const long long n = (long long)c->T * c->H * c->W, rows = (long long)c->B * n;
  const int blocks = static_cast<int>((rows + 7) / 8);
  trace_begin(MATE_K_LN_MODULATE, st);
  if (c->dtype == MATE_BF16)
    ln_modulate_kernel<__nv_bfloat16, 8><<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x),
                                                                  static_cast<__nv_bfloat16*>(h), rows, c->d, n, shift,
                                                                  scale);
  else
    ln_modulate_kernel<float, 4><<<blocks, 256, 0, st>>>(static_cast<const float*>(x), static_cast<float*>(h), rows,
                                                          c->d, n, shift, scale);
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}
}  // namespace

extern "C" {

size_t mate_tesa_backward_workspace_bytes(const mate_config* cfg) {
  if (check_config(cfg) != MATE_OK) return 0;
  const long long items = (long long)(cfg->T / cfg->wt) * (cfg->H / cfg->wh) * (cfg->W / cfg->ww) * cfg->B * cfg->th;
  return (size_t)items * 256 * 2 * sizeof(float) + 256;
}

mate_status tesa_backward(const void* qkv, const void* O, const void* dO, void* dqkv, int shifted,
                          const mate_config* cfg, void* ws, size_t ws_bytes, mate_stream_t stream) {
  MATE_TRY(check_config(cfg));
  if (cfg->dtype != MATE_BF16) return MATE_ERR_UNSUPPORTED;
  if (qkv == nullptr || O == nullptr || dO == nullptr || dqkv == nullptr || ws == nullptr || !aligned16(qkv) ||
      !aligned16(O) || !aligned16(dO) || !aligned16(dqkv) || !aligned16(ws))
    return MATE_ERR_ARG;
  if (ws_bytes < mate_tesa_backward_workspace_bytes(cfg)) return MATE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_launches = 0;
  const int a = cfg->th * cfg->tp;
  const int sft = shifted ? 1 : 0;
  TesaBwdParams p;
  p.qkv = static_cast<const __nv_bfloat16*>(qkv);
  p.ldq = 3 * a;
  p.qcol = 0;
  p.kcol = a;
  p.vcol = 2 * a;
  p.O = static_cast<const __nv_bfloat16*>(O);
  p.dO = static_cast<const __nv_bfloat16*>(dO);
  p.ldo = a;
  p.ocol = 0;
  p.dqkv = static_cast<__nv_bfloat16*>(dqkv);
  p.ldg = 3 * a;
  p.gq = 0;
  p.gk = a;
  p.gv = 2 * a;
  p.stats = static_cast<float*>(ws);
  p.B = cfg->B;
  p.T = cfg->T;
  p.H = cfg->H;
  p.W = cfg->W;
  p.th = cfg->th;
  p.wt = cfg->wt;
  p.wh = cfg->wh;
  p.ww = cfg->ww;
  p.st = sft ? cfg->st : 0;
  p.sh = sft ? cfg->sh : 0;
  p.sw = sft ? cfg->sw : 0;
  p.shifted = sft;
  p.scale = 1.f / std::sqrt(static_cast<float>(cfg->tp));
  p.scale_log2 = 1.4426950408889634f * p.scale;
  const int items = (cfg->T / cfg->wt) * (cfg->H / cfg->wh) * (cfg->W / cfg->ww) * cfg->B * cfg->th;
  const size_t s1 = 1024 + kBdqSmem, s2 = 1024 + kBkvSmem;
  if (!set_smem(tesa_bwd_dq_kernel, s1) || !set_smem(tesa_bwd_dkdv_kernel, s2)) return MATE_ERR_CUDA;
  trace_begin(MATE_K_TESA_BWD_DQ, st);
  tesa_bwd_dq_kernel<<<dim3(items, 2), kTesaBwdThreads, s1, st>>>(p);
  MATE_LAUNCH_CHECK();
  trace_begin(MATE_K_TESA_BWD_DKDV, st);
  tesa_bwd_dkdv_kernel<<<dim3(items, 2), kTesaBwdThreads, s2, st>>>(p);
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

size_t mate_dit_workspace_bytes(const mate_config* cfg) {
  if (check_config(cfg) != MATE_OK || cfg->d > 2048) return 0;
  return plan_dit(cfg, nullptr).bytes;
}

mate_status mate_dit_block_forward(const void* X, const float* c, int dc, const mate_dit_weights* dw,
                                   const mate_weights* mw, int layer_idx, void* Out, const mate_config* cfg, void* ws,
                                   size_t ws_bytes, mate_stream_t stream) {
  MATE_TRY(check_config(cfg));
  if (cfg->d > 2048) return MATE_ERR_UNSUPPORTED;
  if (X == nullptr || c == nullptr || dc <= 0 || dw == nullptr || mw == nullptr || Out == nullptr || ws == nullptr ||
      layer_idx < 0 || dw->W_ada == nullptr || dw->b_ada == nullptr || dw->W1 == nullptr || dw->b1 == nullptr ||
      dw->W2 == nullptr || dw->b2 == nullptr)
    return MATE_ERR_ARG;
  if (!aligned16(X) || !aligned16(Out) || !aligned16(ws) || !aligned16(dw->W1) || !aligned16(dw->W2) ||
      !aligned16(dw->b1) || !aligned16(dw->b2))
    return MATE_ERR_ARG;
  if (X == Out) return MATE_ERR_ARG;
  DitPlan pl = plan_dit(cfg, nullptr);
  if (ws_bytes < pl.bytes) return MATE_ERR_WORKSPACE;
  pl = plan_dit(cfg, ws);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_launches = 0;
  const int d = cfg->d;
  const long long n = (long long)cfg->T * cfg->H * cfg->W, rows = (long long)cfg->B * n;
  // modulation vectors of every sample
  {
    const long long warps = (long long)cfg->B * 6 * d;
    trace_begin(MATE_K_ADA_MODULATION, st);
    if (cfg->dtype == MATE_BF16)
      ada_modulation_kernel<__nv_bfloat16><<<static_cast<int>((warps + 7) / 8), 256, 0, st>>>(
          c, dc, static_cast<const __nv_bfloat16*>(dw->W_ada), dw->b_ada, pl.mod, 6 * d, cfg->B);
    else
      ada_modulation_kernel<float><<<static_cast<int>((warps + 7) / 8), 256, 0, st>>>(
          c, dc, static_cast<const float*>(dw->W_ada), dw->b_ada, pl.mod, 6 * d, cfg->B);
    MATE_LAUNCH_CHECK();
  }
  const float *shift_a = pl.mod, *scale_a = pl.mod + d, *gate_a = pl.mod + 2 * d;
  const float *shift_m = pl.mod + 3 * d, *scale_m = pl.mod + 4 * d, *gate_m = pl.mod + 5 * d;
  // X1 = X + gate_a * MATE(LN(X) (1 + scale_a) + shift_a): the gated residual in the out-projection's epilogue
  MATE_TRY(ln_modulate(cfg, X, pl.h, shift_a, scale_a, st));
  GemmEpilogue mix_ep;
  mix_ep.resid = X;
  mix_ep.ld_resid = d;
  mix_ep.gate = gate_a;
  mix_ep.ld_gate = 6 * d;
  mix_ep.gate_rows = static_cast<int>(n);
  MATE_TRY(forward_impl(pl.h, mw, layer_idx, pl.X1, cfg, pl.mate_ws, pl.mate_bytes, st, nullptr, &mix_ep));
  // Out = X1 + gate_m * MLP(LN(X1) (1 + scale_m) + shift_m)
  MATE_TRY(ln_modulate(cfg, pl.X1, pl.h, shift_m, scale_m, st));
  GemmEpilogue up_ep;
  up_ep.bias = dw->b1;
  up_ep.act = 1;
  GemmEpilogue down_ep;
  down_ep.bias = dw->b2;
  down_ep.resid = pl.X1;
  down_ep.ld_resid = d;
  down_ep.gate = gate_m;
  down_ep.ld_gate = 6 * d;
  down_ep.gate_rows = static_cast<int>(n);
  if (cfg->dtype == MATE_BF16) {
    MATE_TRY(gemm_bf16(MATE_K_MLP_UP, pl.h, d, rows, d, dw->W1, d, 4 * d, pl.Z, 4 * d, nullptr, 0, 0, 0, nullptr, st,
                       nullptr, &up_ep));
    MATE_TRY(gemm_bf16(MATE_K_MLP_DOWN, pl.Z, 4 * d, rows, 4 * d, dw->W2, 4 * d, d, Out, d, nullptr, 0, 0, 0, nullptr,
                       st, nullptr, &down_ep));
  } else {
    MATE_TRY(gemm_f32(MATE_K_MLP_UP, static_cast<const float*>(pl.h), d, rows, d, static_cast<const float*>(dw->W1), d,
                      4 * d, static_cast<float*>(pl.Z), 4 * d, nullptr, 0, 0, 0, nullptr, st, nullptr, &up_ep));
    MATE_TRY(gemm_f32(MATE_K_MLP_DOWN, static_cast<const float*>(pl.Z), 4 * d, rows, 4 * d,
                      static_cast<const float*>(dw->W2), 4 * d, d, static_cast<float*>(Out), d, nullptr, 0, 0, 0,
                      nullptr, st, nullptr, &down_ep));
  }
  return MATE_OK;
}

mate_status mate_device_status(mate_stream_t stream, unsigned int* flags) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MATE_ERR_CUDA;
  // read and clear in one atomic exchange on the device, so that a flag set meanwhile by a kernel on
  // another stream is either returned now or kept for the next call, never lost
  status_take_kernel<<<1, 1, 0, st>>>();
  unsigned int v = 0;
  if (!cuda_ok(cudaGetLastError()) ||
      !cuda_ok(cudaMemcpyFromSymbolAsync(&v, g_dev_status_taken, sizeof(v), 0, cudaMemcpyDeviceToHost, st)) ||
      !cuda_ok(cudaStreamSynchronize(st)))
    return MATE_ERR_CUDA;
  if (flags) *flags = v;
  return v ? MATE_ERR_TIMEOUT : MATE_OK;
}

int mate_last_launch_count(void) { return t_launches; }

mate_status mate_selftest_wait_timeout(unsigned int max_polls, mate_stream_t stream) {
  if (max_polls < 1 || max_polls > 65536) return MATE_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_launches = 0;
  trace_begin(MATE_K_SELFTEST, st);
  wait_timeout_selftest_kernel<<<1, 1, 0, st>>>(max_polls);
  MATE_LAUNCH_CHECK();
  return MATE_OK;
}

mate_status mate_trace_start(int capacity) {
  if (capacity < 0) return MATE_ERR_ARG;
  std::lock_guard<std::mutex> lock(g_trace.mu);
  g_trace.on = false;
  if (static_cast<int>(g_trace.ev.size()) < 2 * capacity) {
    for (size_t e = g_trace.ev.size(); e < static_cast<size_t>(2 * capacity); ++e) {
      cudaEvent_t ev;
      if (cudaEventCreate(&ev) != cudaSuccess) {
        cudaGetLastError();
        return MATE_ERR_CUDA;
      }
      g_trace.ev.push_back(ev);
    }
  }
  g_trace.kid.assign(capacity, -1);
  g_trace.cap = capacity;
  g_trace.n = 0;
  g_trace.on = capacity > 0;
  return MATE_OK;
}

mate_status mate_trace_stop(void) {
  std::lock_guard<std::mutex> lock(g_trace.mu);
  g_trace.on = false;
  return MATE_OK;
}

int mate_trace_read(mate_trace_record* out, int max_records) {
  std::lock_guard<std::mutex> lock(g_trace.mu);
  if (g_trace.on || out == nullptr || max_records < 0) return -1;
  const int n = std::min(g_trace.n, max_records);
  for (int r = 0; r < n; ++r) {
    float ms = 0.f;
    if (cudaEventSynchronize(g_trace.ev[2 * r + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms, g_trace.ev[2 * r], g_trace.ev[2 * r + 1]) != cudaSuccess) {
      cudaGetLastError();
      return -1;
    }
    out[r].kernel = g_trace.kid[r];
    out[r].ms = ms;
  }
  return n;
}

const char* mate_kernel_name(int kernel) {
  switch (kernel) {
    case MATE_K_PACK_WEIGHTS: return "pack_weights";
    case MATE_K_REVIEW_POOL: return "review_pool";
    case MATE_K_IN_PROJ: return "in_projection";
    case MATE_K_IN_PROJ_REVIEW: return "in_projection_review";
    case MATE_K_SOFTPLUS: return "softplus";
    case MATE_K_SSD_GRAM: return "ssd_gram";
    case MATE_K_SSD_STATE: return "ssd_state";
    case MATE_K_SSD_CARRY: return "ssd_carry";
    case MATE_K_SSD_OUTPUT: return "ssd_output";
    case MATE_K_SSD_F32: return "ssd_f32";
    case MATE_K_TESA: return "tesa";
    case MATE_K_TESA_F32: return "tesa_f32";
    case MATE_K_OUT_PROJ: return "out_projection";
    case MATE_K_RMS_GATHER: return "rms_gather";
    case MATE_K_PROJECT: return "project";
    case MATE_K_SCAN_LOCALITY: return "scan_locality";
    case MATE_K_Y_TO_GRID: return "y_to_grid";
    case MATE_K_CONV_SILU: return "conv_silu";
    case MATE_K_GATE_NORM: return "gate_rmsnorm";
    case MATE_K_SSD_BACKWARD: return "ssd_backward_f32";
    case MATE_K_SELFTEST: return "selftest_wait_timeout";
    case MATE_K_ADA_MODULATION: return "ada_modulation";
    case MATE_K_LN_MODULATE: return "ln_modulate";
    case MATE_K_MLP_UP: return "mlp_up";
    case MATE_K_MLP_DOWN: return "mlp_down";
    case MATE_K_TESA_BWD_DQ: return "tesa_backward_dq";
    case MATE_K_TESA_BWD_DKDV: return "tesa_backward_dkdv";
  }
  return "unknown";
}

}  // extern "C"
