/*
 * libmate: forward pass of the LinGen MATE token-mixing block on NVIDIA B200 (sm_100a).
 *
 * Method sources (the pages that describe it):
 *   [ABS]  "Towards High-Resolution Minute-Length Text-to-Video Generation with Linear Computational
 *          Complexity", abstract: MATE replaces DiT self-attention and consists of an MA branch (a
 *          bidirectional Mamba2 block with Rotary Major Scan and review tokens) and a TE branch
 *          (TEmporal Swin Attention).
 *   [NEWS] LinGen news article (weiba1314.com / xihudo.com), section "方法：线性复杂度的 MATE 模块":
 *          RMS unrolls the T x H x W grid with W, H, T as 1st/2nd/3rd priority and swaps priorities
 *          between adjacent layers; TESA is 3D window attention with small fixed windows that slide
 *          between layers; review tokens write an overview of the video tensor into the Mamba hidden
 *          state ahead of the video.
 *   [FEAT] "LinGen：基于Mamba机制的线性复杂度高清长视频生成框架", 关键算法创新: the four RMS modes
 *          (spatial row / spatial column / temporal row / temporal column) and TESA's alternating
 *          normal and shifted windows.
 *
 * Conventions for every entry point
 *   - Tensors are DEVICE pointers owned by the caller, contiguous, channels-last, 16-byte aligned.
 *     Element type follows cfg->dtype (bf16 or fp32) unless the argument says float.
 *   - Calls are stream-ordered on `stream` and never synchronise; they never allocate or free device
 *     memory.  Scratch memory is the caller's workspace `ws` of at least the queried size.
 *   - Host-side validation happens before any launch; a rejected call launches nothing.
 *   - Weight matrices use the out_features x in_features layout (row r = output feature r).
 *   - Layer behaviour is a pure function of layer_idx: scan order layer_idx mod 4, Swin shift on odd
 *     layers.
 *   - The grid token (t, h, w) of sample b is row b*T*H*W + (t*H + h)*W + w of a [B, T, H, W, C]
 *     tensor.
 */
#ifndef MATE_H_
#define MATE_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MATE_API __attribute__((visibility("default")))
#else
#define MATE_API
#endif

/* Same object as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st* mate_stream_t;

typedef enum {
  MATE_OK = 0,
  MATE_ERR_ARG = 1,         /* null pointer, misaligned pointer, order/layer out of range */
  MATE_ERR_SHAPE = 2,       /* inconsistent sizes: window does not divide the grid, bad review count */
  MATE_ERR_WORKSPACE = 3,   /* ws_bytes smaller than the queried workspace size */
  MATE_ERR_CUDA = 4,        /* a CUDA launch or copy failed (cudaGetLastError after the launch) */
  MATE_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out (reported by mate_device_status) */
  MATE_ERR_UNSUPPORTED = 6, /* valid shape that the bf16 tensor-core kernels do not cover */
  MATE_ERR_TOO_LARGE = 7    /* problem needs more scratch than the library's fixed device buffer holds */
} mate_status;

typedef enum { MATE_BF16 = 0, MATE_F32 = 1 } mate_dtype;

/*
 * Block shape.  B samples of a T x H x W latent grid with d channels; Mamba2 with nh heads of size P,
 * state size N, chunk length Q and R review tokens; TESA with th heads of size tp, window
 * (wt, wh, ww) and Swin shift (st, sh, sw) used on odd layers.
 * Requirements: window divides the grid; 0 <= shift < window per axis; R = 16 * Tr with Tr dividing T
 * and 4 dividing H and W (review tokens pool onto a Tr x 4 x 4 grid), R = 0 allowed; d, nh*P, th*tp
 * multiples of 8 elements.
 * bf16 tensor-core path additionally: d % 64 == 0, nh % 8 == 0, P == 64, N == 128, Q == 256,
 * tp == 128, wt*wh*ww == 256.  fp32 path (CUDA-core kernels, for small blocks): P*N <= 1024, tp <= 128.
 * B * (T*H*W + R) < 2^31.
 * mamba_extras = 1 gives the MA branch the rest of a Mamba2 block around the scan: a causal depthwise
 * convolution of width 4 with bias + SiLU on x | B | C (along [review rows; video rows in scan order],
 * zero before each sample's first row, one pass feeding both scan directions), the gate z = W_z X of the
 * video rows and gated RMSNorm  y <- (y silu(z)) / sqrt(mean((y silu(z))^2) + 1e-5) * norm_w  over each
 * row's nh*P channels before the out-projection.  The pages name a Mamba2 block without listing its
 * parts; these are the standard ones.  0 (default): projections and scan only.
 */
typedef struct {
  int B, T, H, W, d;
  int nh, P, N, Q, R;
  int th, tp;
  int wt, wh, ww;
  int st, sh, sw;
  mate_dtype dtype;
  int mamba_extras; /* 0 or 1 */
} mate_config;

/* Block weights, device pointers, caller-owned.  Element type cfg->dtype except the fp32 vectors. */
typedef struct {
  const void* W_in;     /* [nh*P + 2N + nh, d]: output features x (head h at h*P..) | B | C | dt      */
  const float* dt_bias; /* [nh]   delta = softplus(dt + dt_bias)                                     */
  const float* A_log;   /* [nh]   A = -exp(A_log)                                                    */
  const float* D;       /* [nh]   skip weight                                                        */
  const void* W_out;    /* [d, nh*P]  MA out-projection                                              */
  const void* W_qkv;    /* [3*th*tp, d] output features q | k | v, head-major inside each            */
  const void* W_o;      /* [d, th*tp]  TE out-projection                                             */
  /* Optional separate parameters of the backward scan direction (all three or none; null: the backward
   * scan uses dt_bias, A_log and D above).  The pages do not say whether the directions share them. */
  const float* dt_bias_b; /* [nh] */
  const float* A_log_b;   /* [nh] */
  const float* D_b;       /* [nh] */
  /* Required when cfg->mamba_extras = 1, ignored otherwise. */
  const void* W_z;        /* [nh*P, d]  gate projection                                              */
  const float* conv_w;    /* [nh*P + 2N, 4] depthwise taps per channel of x | B | C, tap 3 on the current row */
  const float* conv_b;    /* [nh*P + 2N]  convolution bias                                           */
  const float* norm_w;    /* [nh*P]   gated RMSNorm weight                                           */
  /* Optional: the buffer mate_pack_weights filled from these weights (same cfg, mamba_extras included).
   * Given, mate_forward / mate_forward_host* read the packed projection matrices from it; null, they pack
   * W_in, W_qkv, W_z, W_out and W_o into the workspace on every call. */
  const void* packed;
} mate_weights;

/*
 * The projections run as two GEMMs over packed weight matrices: [W_in; W_qkv (; W_z)] (the MA
 * in-projection fused with TESA's qkv projection, the gate rows last) and [W_out | W_o] (the two
 * out-projections side by side, so that the branch sum falls out of the K reduction).  mate_pack_weights
 * writes both into `packed` (at least mate_packed_weights_bytes(cfg) bytes, 16-byte aligned) once; pass it
 * as w->packed so that the block does not repack on every call.  Stream-ordered; MATE_ERR_ARG for a null
 * or misaligned matrix (W_z required when cfg->mamba_extras = 1), MATE_ERR_WORKSPACE if packed_bytes is
 * too small.  The pages have no counterpart: this is how the fused projections are laid out.
 */
MATE_API size_t mate_packed_weights_bytes(const mate_config* cfg);
MATE_API mate_status mate_pack_weights(const mate_weights* w, const mate_config* cfg, void* packed,
                                       size_t packed_bytes, mate_stream_t stream);

/*
 * Self-test of the timeout report (no counterpart in the pages).  Launches one thread that waits on a
 * device barrier nothing completes, polling at most max_polls times (1 <= max_polls <= 65536), after
 * which it records a timeout in the device status word and returns, as every bounded wait of the library
 * does when it runs out.  The next mate_device_status on the stream then returns MATE_ERR_TIMEOUT and
 * clears the word.  MATE_ERR_ARG if max_polls is out of range.
 */
MATE_API mate_status mate_selftest_wait_timeout(unsigned int max_polls, mate_stream_t stream);

/* Human-readable name of a status code (static string). */
MATE_API const char* mate_status_str(mate_status s);

/* MATE_OK if cfg describes a block this library can run, else the reason (no device work). */
MATE_API mate_status mate_check_config(const mate_config* cfg);

/* Workspace bytes needed by mate_forward / mate_forward_host for this shape (0 if cfg is invalid). */
MATE_API size_t mate_workspace_bytes(const mate_config* cfg);

/* Workspace bytes needed by ssd_scan_bidir for this shape with `prefix_len` prefix rows. */
MATE_API size_t mate_ssd_workspace_bytes(const mate_config* cfg, int prefix_len);

/* Workspace bytes needed by ssd_scan_bidir_pd (separate backward-scan parameters): the backward step
 * sizes, log-decays and review-chunk states come on top of what ssd_scan_bidir needs. */
MATE_API size_t mate_ssd_pd_workspace_bytes(const mate_config* cfg, int prefix_len);

/*
 * Rotary Major Scan reorder ([NEWS] RMS paragraphs; [FEAT] RMS modes).
 *   X  [B, T, H, W, d] -> Xp [B, T*H*W, d] with Xp[b, s_o(t,h,w)] = X[b, t, h, w], where the scan
 *   position s_o unrolls the grid with the order's first-priority axis fastest:
 *     order 0 (spatial row):     s = (t*H + h)*W + w     (W, H, T)
 *     order 1 (spatial column):  s = (t*W + w)*H + h     (H, W, T)
 *     order 2 (temporal row):    s = (h*W + w)*T + t     (T, W, H)
 *     order 3 (temporal column): s = (w*H + h)*T + t     (T, H, W)
 * Bit copy; X and Xp must not overlap.  MATE_ERR_ARG if order is not 0..3.
 */
MATE_API mate_status rms_permute(const void* X, void* Xp, int order, const mate_config* cfg, mate_stream_t stream);

/* Inverse of rms_permute: X[b, t, h, w] = Xp[b, s_o(t,h,w)]. */
MATE_API mate_status rms_unpermute(const void* Xp, void* X, int order, const mate_config* cfg, mate_stream_t stream);

/*
 * Review tokens ([NEWS] review-token paragraph: an overview of the video tensor, written into the
 * Mamba hidden state before the video tokens).  Rv [B, R, d]: the average of X over each cell of the
 * Tr x 4 x 4 pooling grid (cells of (T/Tr) x (H/4) x (W/4) tokens), listed in scan order `order` of
 * that grid.  fp32 accumulation.  Does nothing when R == 0.
 */
MATE_API mate_status review_pool(const void* X, void* Rv, int order, const mate_config* cfg, mate_stream_t stream);

/*
 * Bidirectional Mamba2 selective scan ([ABS] "bidirectional Mamba2 block").  For each sample b the
 * sequence S has L = prefix_len + T*H*W rows: prefix rows first, then the video rows.  Per head h
 * (A_h = -exp(A_log[h]), delta = softplus(dt + dt_bias[h]), zero initial state):
 *     h_t = exp(delta_t A_h) h_{t-1} + delta_t x_t B_t^T,    y_t = h_t C_t + D_h x_t
 * is run over S (forward) and over [prefix rows; video rows reversed] (backward).  The output holds
 * the video rows only: y = y_forward + (y_backward reversed back).
 *   x  [B, L, nh*P]    Bm, Cm [B, L, N]    dt [B, L, nh] float (raw, before softplus)
 *   dt_bias, A_log, D  [nh] float           y [B, T*H*W, nh*P]
 * ws: at least mate_ssd_workspace_bytes(cfg, prefix_len) bytes.  cfg->R is ignored (prefix_len is
 * used instead); prefix_len must satisfy 0 <= prefix_len.
 */
MATE_API mate_status ssd_scan_bidir(const void* x, const void* Bm, const void* Cm, const float* dt, const float* dt_bias,
                           const float* A_log, const float* D, int prefix_len, void* y, const mate_config* cfg,
                           void* ws, size_t ws_bytes, mate_stream_t stream);

/*
 * ssd_scan_bidir with separate parameters for the backward scan direction ([ABS] "bidirectional Mamba2
 * block"; the pages leave open whether the two directions share A, D and the step-size bias).  The
 * forward scan uses dt_bias, A_log, D; the backward scan (over [prefix rows; video rows reversed]) uses
 * delta_b = softplus(dt + dt_bias_b[h]), A_b = -exp(A_log_b[h]) and D_b, with the same x, Bm, Cm and raw
 * dt.  y = y_forward + (y_backward reversed back), each direction including its own D x skip term.
 * With dt_bias_b = dt_bias, A_log_b = A_log, D_b = D it computes what ssd_scan_bidir computes.
 *   dt_bias_b, A_log_b, D_b  [nh] float, device; ws at least mate_ssd_pd_workspace_bytes(cfg, prefix_len)
 *   bytes; every other argument as for ssd_scan_bidir.  MATE_ERR_ARG if any of the three is null;
 *   otherwise the statuses of ssd_scan_bidir.
 */
MATE_API mate_status ssd_scan_bidir_pd(const void* x, const void* Bm, const void* Cm, const float* dt,
                                       const float* dt_bias, const float* A_log, const float* D,
                                       const float* dt_bias_b, const float* A_log_b, const float* D_b,
                                       int prefix_len, void* y, const mate_config* cfg, void* ws, size_t ws_bytes,
                                       mate_stream_t stream);

/*
 * Backward pass of ssd_scan_bidir (training): given the output gradient dy [B, T*H*W, nh*P] of the video
 * rows, the gradients of every input.  The adjoint follows from the forward recurrence by the chain rule
 * (the pages give only the forward computation):
 *     dx, dB, dC  [B, L, nh*P] / [B, L, N]   same layout as x, Bm, Cm (prefix rows included)
 *     ddt         [B, L, nh]  gradient of the raw step input dt (delta = softplus(dt + dt_bias))
 *     ddt_bias, dA_log, dD  [nh]  summed over samples and rows
 * fp32 blocks only (cfg->dtype = MATE_F32; bf16 gives MATE_ERR_UNSUPPORTED); a CUDA-core kernel that
 * keeps every state of one direction in the workspace, for small problems.  ws: at least
 * mate_ssd_backward_workspace_bytes(cfg, prefix_len) bytes.  All gradient outputs are written in full
 * (the summed ones are zeroed first on `stream`).  dB, dC, ddt_bias, dA_log and dD are sums over heads or
 * rows accumulated with float atomics, so their last bits may differ from run to run; dx and ddt are
 * reproducible.
 */
MATE_API size_t mate_ssd_backward_workspace_bytes(const mate_config* cfg, int prefix_len);
MATE_API mate_status ssd_scan_bidir_backward(const void* x, const void* Bm, const void* Cm, const float* dt,
                                             const float* dt_bias, const float* A_log, const float* D,
                                             int prefix_len, const void* dy, void* dx, void* dB, void* dC,
                                             float* ddt, float* ddt_bias, float* dA_log, float* dD,
                                             const mate_config* cfg, void* ws, size_t ws_bytes,
                                             mate_stream_t stream);

/* Size of the fixed device scratch buffer behind ssd_scan_bidir_noalloc: 64 MiB. */
#define MATE_SSD_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * ssd_scan_bidir for callers that must not allocate device memory.  The paper has no counterpart to
 * this entry point; it computes exactly what ssd_scan_bidir computes, with the same arguments minus
 * the workspace.  It exists for callers that are handed their input and output buffers but may not
 * create device allocations of their own: a plugin inside a host framework that owns every device
 * allocation, or a latency-bound serving loop where cudaMalloc and cudaFree would synchronise the
 * device and stall work on other streams.  Such callers can neither size nor own a workspace.
 *
 * Scratch: instead of a caller workspace the scan uses one fixed array of
 * MATE_SSD_NOALLOC_SCRATCH_BYTES bytes in device global memory, part of this library's device code.
 * Every GPU on which the library's device code is loaded holds that array until the process exits.
 * A problem with mate_ssd_workspace_bytes(cfg, prefix_len) > MATE_SSD_NOALLOC_SCRATCH_BYTES is
 * rejected with MATE_ERR_TOO_LARGE before any device work (with the bf16 kernels, nh = 16, B = 1 and
 * 128 prefix rows the scratch takes about 9.4 KiB per video token, which admits up to 26 chunks of 256
 * video tokens, 6 656 tokens; the fp32 kernels need only the step sizes, 4 bytes per row and head).
 *
 * Set-up: the first call on a device (the device current at the call) looks up the array's device
 * address once, which can load the library's device code onto that device; make that first call
 * before any stream capture on the device.  Later calls on the device reuse the address as long as the
 * device's CUDA context is the same one; after cudaDeviceReset the next call looks it up again (and is
 * then again a first call).
 *
 * Sharing: all calls on one device use the same array, and it keeps what the last call left in it.
 * Each call writes every scratch byte it reads before reading it, so nothing needs clearing between
 * calls.  Calls whose executions overlap on the GPU (on streams with no ordering between them, from
 * one host thread or several) race on the array and give wrong results; calls on one stream run one
 * after the other and are safe.
 *
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine is called.  Errors as
 * ssd_scan_bidir, plus MATE_ERR_TOO_LARGE (checked before the pointers); MATE_ERR_CUDA if the address
 * look-up fails.
 */
MATE_API mate_status ssd_scan_bidir_noalloc(const void* x, const void* Bm, const void* Cm, const float* dt,
                                            const float* dt_bias, const float* A_log, const float* D, int prefix_len,
                                            void* y, const mate_config* cfg, mate_stream_t stream);

/*
 * TEmporal Swin Attention ([NEWS] TESA paragraph; [FEAT] TESA): window attention on qkv
 * [B, T, H, W, 3*th*tp] (q | k | v, head-major) -> O [B, T, H, W, th*tp].  shifted == 0: windows
 * (wt, wh, ww) tile the grid.  shifted != 0: the grid is rolled by -(st, sh, sw) before tiling and
 * rolled back after; keys that wrapped around an axis and keys that did not are masked from each other.
 * Per window and head: softmax(q k^T / sqrt(tp)) v with fp32 softmax.
 */
MATE_API mate_status tesa_forward(const void* qkv, void* O, int shifted, const mate_config* cfg, mate_stream_t stream);

/*
 * Backward pass of tesa_forward (training; the pages give only the forward computation, and its gradient
 * follows by the chain rule).  Given the forward's input qkv, its output O and the output gradient dO
 * (all [B, T, H, W, .] as for tesa_forward, heads in the same column order), writes dqkv [B, T, H, W,
 * 3*th*tp] (dq | dk | dv in the column layout of qkv).  Per window and head, with P the forward's masked
 * softmax of q k^T / sqrt(tp):
 *     dv = P^T dO,   dP = dO v^T,   dS = P (dP - rowsum(dO * O)),   dq = dS k / sqrt(tp),   dk = dS^T q / sqrt(tp).
 * Every token belongs to exactly one window per layer, so each row of dqkv is written once.  bf16 blocks
 * only (MATE_ERR_UNSUPPORTED otherwise); tensor-core products on fp16 operands (q, k, v and dO converted
 * exactly, P and dS rounded to fp16, values beyond the fp16 range saturating) and fp32 softmax statistics.  ws: at least mate_tesa_backward_workspace_bytes(cfg) bytes (per window,
 * head and query: the softmax normaliser and rowsum(dO * O), written by the first kernel, read by the second).
 */
MATE_API size_t mate_tesa_backward_workspace_bytes(const mate_config* cfg);
MATE_API mate_status tesa_backward(const void* qkv, const void* O, const void* dO, void* dqkv, int shifted,
                                   const mate_config* cfg, void* ws, size_t ws_bytes, mate_stream_t stream);

/*
 * Scan locality ([NEWS] method, Rotary Major Scan paragraphs; [FEAT] 功能特色 / RMS: the alternating
 * orders bring the average distance, after the scan, between originally adjacent tokens down to the level
 * of Zigzag and Hilbert scans).  Over all pairs of tokens of a T x H x W grid that differ by one step along
 * one axis, the distance of their positions in the sequence of index map `map`:
 *   0..3  the Rotary Major Scan orders (as rms_permute);
 *   4     Zigzag: 3D boustrophedon (w fastest, reversing on every (t, h) line; h reversing on every t plane);
 *   5     Hilbert: cubes of side H = W stacked along t, each along the 3D Hilbert curve; needs H = W a power
 *         of two dividing T (MATE_ERR_UNSUPPORTED otherwise);
 *   6     the four orders' rotation: per pair the smallest distance over the four orders.
 * out: DEVICE array of 3 unsigned long long (8-byte aligned), overwritten on `stream` with the sum of the
 * distances, the number of pairs and the largest distance.  Integer arithmetic: exact.
 */
MATE_API mate_status mate_scan_locality(int T, int H, int W, int map, unsigned long long* out, mate_stream_t stream);

/*
 * Tensor-core projection used by the block's in/out maps: C[M, N] = A[M, K] W[N, K]^T in bf16 with
 * fp32 accumulation (row strides lda, ldw, ldc in elements, multiples of 8; K a multiple of 64).
 * bf16 only (cfg is not needed); MATE_ERR_UNSUPPORTED otherwise.
 */
MATE_API mate_status mate_project_bf16(const void* A, int lda, long long M, int K, const void* Wt, int ldw, int N,
                                       void* C, int ldc, mate_stream_t stream);

/*
 * The MATE block: Out = MA(X) + TE(X) for X, Out [B, T, H, W, d] (may not alias).  Layer layer_idx >= 0
 * selects scan order layer_idx mod 4 and the Swin shift on odd layers.
 *   MA: review tokens (pooled from X, in scan order) prefixed to the scanned sequence; in-projection
 *       W_in; bidirectional scan; out-projection W_out of the video rows; back to grid order.
 *   TE: qkv = X W_qkv^T; tesa; projection W_o.
 * ws: at least mate_workspace_bytes(cfg) bytes (caller-owned, no alignment beyond 256 bytes needed).
 */
MATE_API mate_status mate_forward(const void* X, const mate_weights* w, int layer_idx, void* Out, const mate_config* cfg,
                         void* ws, size_t ws_bytes, mate_stream_t stream);

/*
 * mate_forward with HOST input and output: copies X_host (B*T*H*W*d elements) to the device part of
 * the workspace, runs the block and copies Out back to Out_host (page-locked host buffers give
 * full-speed asynchronous copies).  For bf16 blocks the copies go in four row chunks on two copy streams
 * of the library's own (one pair per device, created on the first call): the in-projection of a chunk
 * starts as soon as it has landed, and each chunk of Out leaves as soon as its out-projection is done.
 * The copies start after all earlier work on `stream`, and the call ends on `stream` only when the last
 * chunk has reached Out_host.  The host buffers must stay valid until the stream reaches the end of the
 * call.  ws: at least mate_forward_host_workspace_bytes(cfg) bytes.
 */
MATE_API mate_status mate_forward_host(const void* X_host, const mate_weights* w, int layer_idx, void* Out_host,
                              const mate_config* cfg, void* ws, size_t ws_bytes, mate_stream_t stream);

/*
 * mate_forward_host for a sequence of calls on one workspace in which a call's host copies overlap the
 * neighbouring calls' work: its input copy runs during the previous call's output copy (the two
 * directions of the host link at the same time), and its output copy runs during the next call's block.
 * Same arguments and result as mate_forward_host; calls alternate between two device input slots and two
 * device output slots of the workspace.  Ordering:
 *   - A call's input copy waits only until the call before the previous one (same slot) has read its
 *     input, and for the output copies of the two previous calls whose Out_host overlaps X_host (so a
 *     chain that feeds one call's output to the next call as input stays correct).  It does NOT wait for
 *     other work enqueued on `stream` before the call: if device work on `stream` writes X_host (a
 *     device-to-host copy), synchronise before the call.  The first call on a workspace, and a call after
 *     calls on another workspace of the same device, start their copies after all earlier work on `stream`.
 *   - When `stream` reaches the end of a call, the PREVIOUS pipelined call's Out_host is complete; this
 *     call's Out_host is complete when `stream` reaches the end of the next pipelined call or of a
 *     mate_forward_host_flush.  mate_forward_host (the one-at-a-time form) waits for all of them first.
 * For bf16 blocks; fp32 blocks run as mate_forward_host.  The pages have no counterpart.
 */
MATE_API mate_status mate_forward_host_pipelined(const void* X_host, const mate_weights* w, int layer_idx,
                                                 void* Out_host, const mate_config* cfg, void* ws, size_t ws_bytes,
                                                 mate_stream_t stream);

/* Makes `stream` wait for the output copies of every pipelined call on the current device that no stream
 * waits for yet; once `stream` reaches this point, every such call's Out_host is complete. */
MATE_API mate_status mate_forward_host_flush(mate_stream_t stream);

/* Workspace bytes needed by mate_forward_host and mate_forward_host_pipelined: the block's workspace,
 * two device input slots and two device output slots. */
MATE_API size_t mate_forward_host_workspace_bytes(const mate_config* cfg);

/*
 * A DiT block with the MATE block as its token mixer ([ABS]: MATE replaces the self-attention of a DiT;
 * [NEWS] method: the rest of the DiT stays as it is).  The pages do not describe that rest; this is the
 * standard DiT block with adaLN-Zero conditioning:
 *   [shift_a, scale_a, gate_a, shift_m, scale_m, gate_m] = silu(c_b) W_ada^T + b_ada   (sample b, 6 x d)
 *   X1  = X  + gate_a * MATE(LN(X)  (1 + scale_a) + shift_a)          (MATE: mate_forward, layer_idx)
 *   Out = X1 + gate_m * (W2 gelu_tanh(W1 (LN(X1) (1 + scale_m) + shift_m) + b1) + b2)
 * LN: per token over d channels, no affine parameters, eps 1e-6; gelu_tanh(v) = v/2 (1 + tanh(sqrt(2/pi)
 * (v + 0.044715 v^3))); no cross-attention (text enters through c).  The gated residuals are applied in the
 * epilogues of the out-projection and of the MLP's second GEMM; the GELU in the first GEMM's epilogue.
 *   X, Out [B, T, H, W, d] cfg->dtype (may not alias); c [B, dc] float; d <= 2048.
 *   dw: W_ada [6d, dc], W1 [4d, d], W2 [d, 4d] in cfg->dtype; b_ada [6d], b1 [4d], b2 [d] float.
 *   mw: the mixer's weights as for mate_forward (mw->packed may hold mate_pack_weights' buffer).
 * ws: at least mate_dit_workspace_bytes(cfg) bytes.  MATE_ERR_UNSUPPORTED for d > 2048.
 */
typedef struct {
  const void* W_ada;   /* [6d, dc] */
  const float* b_ada;  /* [6d] */
  const void* W1;      /* [4d, d] */
  const float* b1;     /* [4d] */
  const void* W2;      /* [d, 4d] */
  const float* b2;     /* [d] */
} mate_dit_weights;

MATE_API size_t mate_dit_workspace_bytes(const mate_config* cfg);
MATE_API mate_status mate_dit_block_forward(const void* X, const float* c, int dc, const mate_dit_weights* dw,
                                            const mate_weights* mw, int layer_idx, void* Out, const mate_config* cfg,
                                            void* ws, size_t ws_bytes, mate_stream_t stream);

/*
 * Reads and clears the device status word that kernels set when a bounded wait runs out.  Synchronises
 * `stream` first, then takes the word with one atomic exchange on the device (a flag that a kernel on
 * another stream sets meanwhile is reported now or by the next call, never dropped), and synchronises
 * `stream` again.  *flags receives the raw bits (1 = wait timed out); returns MATE_ERR_TIMEOUT if any bit
 * was set, MATE_OK otherwise.
 */
MATE_API mate_status mate_device_status(mate_stream_t stream, unsigned int* flags);

/* Number of kernel launches the last successful mate_forward call issued on this thread. */
MATE_API int mate_last_launch_count(void);

/*
 * Kernel timing trace (an instrumentation aid; the pages have no counterpart).  Between
 * mate_trace_start(capacity) and mate_trace_stop(), each kernel launch of this library (up to `capacity`
 * launches, from any thread) records a CUDA event on its stream just before and just after the launch.
 * mate_trace_read then waits for those events and writes, per launch in launch order, the kernel's
 * identity and its device duration in milliseconds; it returns the number of records (-1 while a trace
 * is on or on a CUDA error).  Starting a trace discards the previous one.  Events are created on the
 * device current at mate_trace_start, so launches must run on that device; they are kept for reuse.
 * The events add a few microseconds of host work per launch and nothing to the kernels themselves.
 */
typedef enum {
  MATE_K_PACK_WEIGHTS = 0,     /* packing [W_in; W_qkv] and [W_out | W_o] */
  MATE_K_REVIEW_POOL = 1,
  MATE_K_IN_PROJ = 2,          /* fused MA in-projection + TESA qkv projection of the video rows */
  MATE_K_IN_PROJ_REVIEW = 3,   /* MA in-projection of the review rows */
  MATE_K_SOFTPLUS = 4,         /* delta = softplus(dt + dt_bias), standalone scan only */
  MATE_K_SSD_GRAM = 5,
  MATE_K_SSD_STATE = 6,
  MATE_K_SSD_CARRY = 7,
  MATE_K_SSD_OUTPUT = 8,
  MATE_K_SSD_F32 = 9,
  MATE_K_TESA = 10,
  MATE_K_TESA_F32 = 11,
  MATE_K_OUT_PROJ = 12,        /* fused out-projection [y | O] [W_out | W_o]^T (the branch sum) */
  MATE_K_RMS_GATHER = 13,
  MATE_K_PROJECT = 14,         /* mate_project_bf16 */
  MATE_K_SCAN_LOCALITY = 15,   /* mate_scan_locality */
  MATE_K_Y_TO_GRID = 16,       /* scan-order y rows back to grid order (time-fastest scan orders) */
  MATE_K_CONV_SILU = 17,       /* causal depthwise convolution + SiLU on x | B | C (mamba_extras) */
  MATE_K_GATE_NORM = 18,       /* y silu(z) and gated RMSNorm (mamba_extras) */
  MATE_K_SSD_BACKWARD = 19,    /* ssd_scan_bidir_backward (fp32) */
  MATE_K_SELFTEST = 20,        /* mate_selftest_wait_timeout */
  MATE_K_ADA_MODULATION = 21,  /* DiT block: modulation vectors silu(c) W_ada^T + b_ada */
  MATE_K_LN_MODULATE = 22,     /* DiT block: layer norm + scale and shift */
  MATE_K_MLP_UP = 23,          /* DiT block: gelu(h W1^T + b1) */
  MATE_K_MLP_DOWN = 24,        /* DiT block: X1 + gate_m (Z W2^T + b2) */
  MATE_K_TESA_BWD_DQ = 25,     /* tesa_backward: row statistics, delta and dQ */
  MATE_K_TESA_BWD_DKDV = 26    /* tesa_backward: dK and dV */
} mate_kernel;

typedef struct {
  int kernel;   /* a mate_kernel value */
  float ms;     /* device time between the events around the launch */
} mate_trace_record;

MATE_API mate_status mate_trace_start(int capacity);
MATE_API mate_status mate_trace_stop(void);
MATE_API int mate_trace_read(mate_trace_record* out, int max_records);
MATE_API const char* mate_kernel_name(int kernel);

#ifdef __cplusplus
}
#endif
#endif /* MATE_H_ */
