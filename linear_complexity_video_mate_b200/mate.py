"""Python binding of libmate: argument marshalling only.

Every step of the MATE block runs in the CUDA library (include/mate.h); PyTorch provides device memory
and the current stream.  There is no Python or CPU implementation behind these calls: if libmate.so is
missing, the first call raises ImportError.
"""
from __future__ import annotations

import ctypes
from typing import Dict, Optional

import torch

from . import _lib

__all__ = ["MateBlock", "DitBlock", "dit_weights_to_device", "rms_permute", "rms_unpermute", "review_pool", "ssd_scan_bidir", "ssd_scan_bidir_pd",
           "ssd_scan_bidir_noalloc", "ssd_scan_bidir_backward", "tesa_forward", "tesa_backward", "project_bf16", "device_status",
           "torch_dtype", "weights_to_device", "scan_locality", "KernelTrace"]


def torch_dtype(cfg) -> torch.dtype:
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, dtype: torch.dtype, numel: int, name: str):
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous() or t.numel() != numel:
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor with {numel} elements, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


def weights_to_device(w: Dict, cfg, device="cuda") -> Dict[str, torch.Tensor]:
    """Host weight arrays (numpy / tensors) -> device tensors in the library's dtypes."""
    dt = torch_dtype(cfg)
    out = {}
    for k in ("W_in", "W_out", "W_qkv", "W_o", "W_z"):
        if k in w:   # W_z: the optional gate projection of the full Mamba2 block
            out[k] = torch.as_tensor(w[k]).to(device=device, dtype=dt).contiguous()
    for k in ("dt_bias", "A_log", "D", "dt_bias_b", "A_log_b", "D_b", "conv_w", "conv_b", "norm_w"):
        if k in w:   # optional: the backward-scan parameters, the convolution and the norm weight
            out[k] = torch.as_tensor(w[k]).to(device=device, dtype=torch.float32).contiguous()
    return out


class MateBlock:
    """One MATE block (MA + TE branches) with its weights resident on the GPU and a reusable workspace.
    Weights W_z, conv_w, conv_b and norm_w, given together, make the MA branch's core a full Mamba2 block
    (causal convolution + SiLU on x | B | C, SiLU(z) gate, gated RMSNorm).  The projection matrices are
    packed once here (mate_pack_weights); pack=False makes every forward pack them again instead."""

    def __init__(self, cfg, weights: Dict[str, torch.Tensor], device="cuda", pack: bool = True,
                 workspace: bool = True):
        lib = _lib.load()
        self.cfg = cfg
        ext = [k for k in ("W_z", "conv_w", "conv_b", "norm_w") if k in weights]
        if ext and len(ext) != 4:
            raise ValueError(f"Mamba2 extras: give W_z, conv_w, conv_b and norm_w together, got {ext}")
        self.extras = bool(ext)
        self.ccfg = _lib.make_config(cfg, self.extras)
        _lib.check(lib.mate_check_config(ctypes.byref(self.ccfg)), "mate_check_config")
        self.device = torch.device(device)
        self.dtype = torch_dtype(cfg)
        self.w = weights
        n_in = cfg.nh * cfg.P + 2 * cfg.N + cfg.nh
        _need(weights["W_in"], self.dtype, n_in * cfg.d, "W_in")
        _need(weights["W_out"], self.dtype, cfg.d * cfg.nh * cfg.P, "W_out")
        _need(weights["W_qkv"], self.dtype, 3 * cfg.th * cfg.tp * cfg.d, "W_qkv")
        _need(weights["W_o"], self.dtype, cfg.d * cfg.th * cfg.tp, "W_o")
        for k in ("dt_bias", "A_log", "D"):
            _need(weights[k], torch.float32, cfg.nh, k)
        bwd = [k for k in ("dt_bias_b", "A_log_b", "D_b") if k in weights]
        if bwd and len(bwd) != 3:
            raise ValueError(f"backward-scan parameters: give dt_bias_b, A_log_b and D_b together, got {bwd}")
        for k in bwd:
            _need(weights[k], torch.float32, cfg.nh, k)
        if self.extras:
            nP, Cx = cfg.nh * cfg.P, cfg.nh * cfg.P + 2 * cfg.N
            _need(weights["W_z"], self.dtype, nP * cfg.d, "W_z")
            _need(weights["conv_w"], torch.float32, Cx * 4, "conv_w")
            _need(weights["conv_b"], torch.float32, Cx, "conv_b")
            _need(weights["norm_w"], torch.float32, nP, "norm_w")
        self.cw = _lib.CWeights(*(weights[k].data_ptr() if k in weights else None for k in
                                  ("W_in", "dt_bias", "A_log", "D", "W_out", "W_qkv", "W_o", "dt_bias_b", "A_log_b",
                                   "D_b", "W_z", "conv_w", "conv_b", "norm_w")))
        self.packed = None
        if pack:
            nb = lib.mate_packed_weights_bytes(ctypes.byref(self.ccfg))
            self.packed = torch.empty(nb, dtype=torch.uint8, device=self.device)
            _lib.check(lib.mate_pack_weights(ctypes.byref(self.cw), ctypes.byref(self.ccfg), _p(self.packed), nb,
                                             _s(None)), "mate_pack_weights")
            self.cw.packed = self.packed.data_ptr()
        self.ws_bytes = lib.mate_workspace_bytes(ctypes.byref(self.ccfg))
        self.ws = torch.empty(self.ws_bytes if workspace else 0, dtype=torch.uint8, device=self.device)
        self.ws_host = None
        self.numel = cfg.B * cfg.T * cfg.H * cfg.W * cfg.d

    def forward(self, X: torch.Tensor, layer_idx: int, out: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """Out = MA(X) + TE(X) for X [B, T, H, W, d] on the GPU (stream-ordered, no synchronisation)."""
        _need(X, self.dtype, self.numel, "X")
        if out is None:
            out = torch.empty_like(X)
        _need(out, self.dtype, self.numel, "out")
        st = _lib.load().mate_forward(_p(X), ctypes.byref(self.cw), int(layer_idx), _p(out), ctypes.byref(self.ccfg),
                                      _p(self.ws), self.ws_bytes, _s(stream))
        _lib.check(st, "mate_forward")
        return out

    def forward_host(self, X_host: torch.Tensor, layer_idx: int, out_host: torch.Tensor,
                     stream: Optional[torch.cuda.Stream] = None, pipelined: bool = False) -> torch.Tensor:
        """mate_forward_host: host (page-locked) input and output, copies inside the call.  pipelined: the copies
        overlap the neighbouring calls' work (mate_forward_host_pipelined); out_host is then complete once the
        stream reaches the end of the next pipelined call or of flush_host()."""
        lib = _lib.load()
        if self.ws_host is None:
            nb = lib.mate_forward_host_workspace_bytes(ctypes.byref(self.ccfg))
            self.ws_host = torch.empty(nb, dtype=torch.uint8, device=self.device)
        for t, nm in ((X_host, "X_host"), (out_host, "out_host")):
            if t.is_cuda or t.dtype != self.dtype or t.numel() != self.numel or not t.is_contiguous():
                raise ValueError(f"{nm}: expected a contiguous host {self.dtype} tensor with {self.numel} elements")
        fn = lib.mate_forward_host_pipelined if pipelined else lib.mate_forward_host
        st = fn(_p(X_host), ctypes.byref(self.cw), int(layer_idx), _p(out_host), ctypes.byref(self.ccfg),
                _p(self.ws_host), self.ws_host.numel(), _s(stream))
        _lib.check(st, "mate_forward_host_pipelined" if pipelined else "mate_forward_host")
        return out_host

    @staticmethod
    def flush_host(stream: Optional[torch.cuda.Stream] = None):
        """mate_forward_host_flush: the stream waits for every pipelined call's output copy."""
        _lib.check(_lib.load().mate_forward_host_flush(_s(stream)), "mate_forward_host_flush")

    @staticmethod
    def last_launch_count() -> int:
        return _lib.load().mate_last_launch_count()


def dit_weights_to_device(w: Dict, cfg, device="cuda") -> Dict[str, torch.Tensor]:
    """Host DiT-block weights (W_ada [6d, dc], W1 [4d, d], W2 [d, 4d], b_ada, b1, b2) -> device tensors in the
    library's dtypes (matrices in the block's dtype, biases fp32)."""
    dt = torch_dtype(cfg)
    out = {k: torch.as_tensor(w[k]).to(device=device, dtype=dt).contiguous() for k in ("W_ada", "W1", "W2")}
    out.update({k: torch.as_tensor(w[k]).to(device=device, dtype=torch.float32).contiguous()
                for k in ("b_ada", "b1", "b2")})
    return out


class DitBlock:
    """A DiT block with the MATE block as its token mixer (mate_dit_block_forward): adaLN-Zero modulation
    from a per-sample conditioning vector c [B, dc], the mixer behind a gated residual, and a gated GELU MLP
    of width 4 d."""

    def __init__(self, cfg, mate_weights: Dict[str, torch.Tensor], dit_weights: Dict[str, torch.Tensor], dc: int,
                 device="cuda"):
        lib = _lib.load()
        self.cfg, self.dc = cfg, int(dc)
        self.mix = MateBlock(cfg, mate_weights, device, workspace=False)
        d = cfg.d
        dt = torch_dtype(cfg)
        _need(dit_weights["W_ada"], dt, 6 * d * self.dc, "W_ada")
        _need(dit_weights["W1"], dt, 4 * d * d, "W1")
        _need(dit_weights["W2"], dt, 4 * d * d, "W2")
        _need(dit_weights["b_ada"], torch.float32, 6 * d, "b_ada")
        _need(dit_weights["b1"], torch.float32, 4 * d, "b1")
        _need(dit_weights["b2"], torch.float32, d, "b2")
        self.w = dit_weights
        self.cw = _lib.CDitWeights(*(dit_weights[k].data_ptr() for k in ("W_ada", "b_ada", "W1", "b1", "W2", "b2")))
        self.ws_bytes = lib.mate_dit_workspace_bytes(ctypes.byref(self.mix.ccfg))
        if self.ws_bytes == 0:
            raise ValueError("mate_dit_workspace_bytes: configuration not supported by the DiT block")
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)

    def forward(self, X: torch.Tensor, c: torch.Tensor, layer_idx: int, out: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        _need(X, self.mix.dtype, self.mix.numel, "X")
        _need(c, torch.float32, self.cfg.B * self.dc, "c")
        if out is None:
            out = torch.empty_like(X)
        _need(out, self.mix.dtype, self.mix.numel, "out")
        st = _lib.load().mate_dit_block_forward(_p(X), _p(c), self.dc, ctypes.byref(self.cw),
                                                ctypes.byref(self.mix.cw), int(layer_idx), _p(out),
                                                ctypes.byref(self.mix.ccfg), _p(self.ws), self.ws_bytes, _s(stream))
        _lib.check(st, "mate_dit_block_forward")
        return out


def _cfg(cfg):
    c = _lib.make_config(cfg)
    return c


def rms_permute(X: torch.Tensor, order: int, cfg, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    n = cfg.T * cfg.H * cfg.W
    if out is None:
        out = torch.empty((cfg.B, n, cfg.d), dtype=X.dtype, device=X.device)
    c = _cfg(cfg)
    _lib.check(_lib.load().rms_permute(_p(X), _p(out), int(order), ctypes.byref(c), _s(stream)), "rms_permute")
    return out


def rms_unpermute(Xp: torch.Tensor, order: int, cfg, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.W, cfg.d), dtype=Xp.dtype, device=Xp.device)
    c = _cfg(cfg)
    _lib.check(_lib.load().rms_unpermute(_p(Xp), _p(out), int(order), ctypes.byref(c), _s(stream)), "rms_unpermute")
    return out


def review_pool(X: torch.Tensor, order: int, cfg, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((cfg.B, cfg.R, cfg.d), dtype=X.dtype, device=X.device)
    c = _cfg(cfg)
    _lib.check(_lib.load().review_pool(_p(X), _p(out), int(order), ctypes.byref(c), _s(stream)), "review_pool")
    return out


def ssd_scan_bidir(x, Bm, Cm, dt, dt_bias, A_log, D, prefix_len: int, cfg, out=None, ws=None, stream=None):
    """Bidirectional selective scan over [prefix; video] rows: x [B, L, nh*P], Bm/Cm [B, L, N], dt [B, L, nh]
    (fp32, before softplus).  Returns y [B, T*H*W, nh*P] for the video rows."""
    lib = _lib.load()
    c = _cfg(cfg)
    n = cfg.T * cfg.H * cfg.W
    if out is None:
        out = torch.empty((cfg.B, n, cfg.nh * cfg.P), dtype=x.dtype, device=x.device)
    nb = lib.mate_ssd_workspace_bytes(ctypes.byref(c), int(prefix_len))
    if ws is None or ws.numel() < nb:
        ws = torch.empty(nb, dtype=torch.uint8, device=x.device)
    st = lib.ssd_scan_bidir(_p(x), _p(Bm), _p(Cm), _p(dt), _p(dt_bias), _p(A_log), _p(D), int(prefix_len), _p(out),
                            ctypes.byref(c), _p(ws), ws.numel(), _s(stream))
    _lib.check(st, "ssd_scan_bidir")
    return out


def ssd_scan_bidir_pd(x, Bm, Cm, dt, dt_bias, A_log, D, dt_bias_b, A_log_b, D_b, prefix_len: int, cfg, out=None,
                      ws=None, stream=None):
    """ssd_scan_bidir with the backward scan's own step-size bias, A_log and D ([nh] fp32 each)."""
    lib = _lib.load()
    c = _cfg(cfg)
    n = cfg.T * cfg.H * cfg.W
    if out is None:
        out = torch.empty((cfg.B, n, cfg.nh * cfg.P), dtype=x.dtype, device=x.device)
    nb = lib.mate_ssd_pd_workspace_bytes(ctypes.byref(c), int(prefix_len))
    if ws is None or ws.numel() < nb:
        ws = torch.empty(nb, dtype=torch.uint8, device=x.device)
    st = lib.ssd_scan_bidir_pd(_p(x), _p(Bm), _p(Cm), _p(dt), _p(dt_bias), _p(A_log), _p(D), _p(dt_bias_b),
                               _p(A_log_b), _p(D_b), int(prefix_len), _p(out), ctypes.byref(c), _p(ws), ws.numel(),
                               _s(stream))
    _lib.check(st, "ssd_scan_bidir_pd")
    return out


def ssd_scan_bidir_backward(x, Bm, Cm, dt, dt_bias, A_log, D, dy, prefix_len: int, cfg, ws=None, stream=None):
    """Gradients of ssd_scan_bidir (fp32 blocks) given the video rows' output gradient dy [B, T*H*W, nh*P]:
    a dict with dx, dB, dC (layouts of x, Bm, Cm), ddt (layout of dt) and ddt_bias, dA_log, dD [nh]."""
    lib = _lib.load()
    c = _cfg(cfg)
    L = cfg.n + int(prefix_len)
    for t, nm, numel in ((x, "x", cfg.B * L * cfg.nh * cfg.P), (Bm, "Bm", cfg.B * L * cfg.N),
                         (Cm, "Cm", cfg.B * L * cfg.N), (dt, "dt", cfg.B * L * cfg.nh),
                         (dy, "dy", cfg.B * cfg.n * cfg.nh * cfg.P), (dt_bias, "dt_bias", cfg.nh),
                         (A_log, "A_log", cfg.nh), (D, "D", cfg.nh)):
        _need(t, torch.float32, numel, nm)
    f32 = dict(dtype=torch.float32, device=x.device)
    g = dict(dx=torch.empty_like(x), dB=torch.empty_like(Bm), dC=torch.empty_like(Cm), ddt=torch.empty_like(dt),
             ddt_bias=torch.empty(cfg.nh, **f32), dA_log=torch.empty(cfg.nh, **f32), dD=torch.empty(cfg.nh, **f32))
    nb = lib.mate_ssd_backward_workspace_bytes(ctypes.byref(c), int(prefix_len))
    if ws is None or ws.numel() < nb:
        ws = torch.empty(nb, dtype=torch.uint8, device=x.device)
    st = lib.ssd_scan_bidir_backward(_p(x), _p(Bm), _p(Cm), _p(dt), _p(dt_bias), _p(A_log), _p(D), int(prefix_len),
                                     _p(dy), _p(g["dx"]), _p(g["dB"]), _p(g["dC"]), _p(g["ddt"]), _p(g["ddt_bias"]),
                                     _p(g["dA_log"]), _p(g["dD"]), ctypes.byref(c), _p(ws), ws.numel(), _s(stream))
    _lib.check(st, "ssd_scan_bidir_backward")
    return g


def ssd_scan_bidir_noalloc(x, Bm, Cm, dt, dt_bias, A_log, D, prefix_len: int, cfg, out, stream=None):
    """ssd_scan_bidir on the library's fixed device scratch, for callers that may not allocate device memory.
    Nothing is allocated here either: the caller passes the output `out` [B, T*H*W, nh*P]."""
    c = _cfg(cfg)
    st = _lib.load().ssd_scan_bidir_noalloc(_p(x), _p(Bm), _p(Cm), _p(dt), _p(dt_bias), _p(A_log), _p(D),
                                            int(prefix_len), _p(out), ctypes.byref(c), _s(stream))
    _lib.check(st, "ssd_scan_bidir_noalloc")
    return out


def tesa_forward(qkv: torch.Tensor, shifted: bool, cfg, out: Optional[torch.Tensor] = None, stream=None):
    if out is None:
        out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.W, cfg.th * cfg.tp), dtype=qkv.dtype, device=qkv.device)
    c = _cfg(cfg)
    _lib.check(_lib.load().tesa_forward(_p(qkv), _p(out), int(bool(shifted)), ctypes.byref(c), _s(stream)),
               "tesa_forward")
    return out


def tesa_backward(qkv: torch.Tensor, O: torch.Tensor, dO: torch.Tensor, shifted: bool, cfg, out=None, ws=None,
                  stream=None) -> torch.Tensor:
    """Gradient of tesa_forward with respect to qkv [B, T, H, W, 3 th tp], given its output O and the output
    gradient dO [B, T, H, W, th tp] (bf16 blocks)."""
    lib = _lib.load()
    c = _cfg(cfg)
    a = cfg.th * cfg.tp
    n = cfg.B * cfg.T * cfg.H * cfg.W
    _need(qkv, torch.bfloat16, n * 3 * a, "qkv")
    _need(O, torch.bfloat16, n * a, "O")
    _need(dO, torch.bfloat16, n * a, "dO")
    if out is None:
        out = torch.empty_like(qkv)
    nb = lib.mate_tesa_backward_workspace_bytes(ctypes.byref(c))
    if ws is None or ws.numel() < nb:
        ws = torch.empty(nb, dtype=torch.uint8, device=qkv.device)
    _lib.check(lib.tesa_backward(_p(qkv), _p(O), _p(dO), _p(out), int(bool(shifted)), ctypes.byref(c), _p(ws),
                                 ws.numel(), _s(stream)), "tesa_backward")
    return out


def project_bf16(A: torch.Tensor, Wt: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """C = A W^T on tensor cores: A [M, K] bf16, Wt [N, K] bf16 -> C [M, N] bf16."""
    M, K = A.shape
    N = Wt.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=A.device)
    st = _lib.load().mate_project_bf16(_p(A), A.stride(0), M, K, _p(Wt), Wt.stride(0), N, _p(out), out.stride(0),
                                       _s(stream))
    _lib.check(st, "mate_project_bf16")
    return out


def device_status(stream=None) -> int:
    """Synchronise and read/clear the device status word (1 = a bounded wait ran out)."""
    flags = ctypes.c_uint(0)
    _lib.load().mate_device_status(_s(stream), ctypes.byref(flags))
    return int(flags.value)


class KernelTrace:
    """Per-launch device times of this library's kernels between start() and stop() (CUDA events around
    each launch, recorded by the library).  read() -> list of (kernel name, ms) in launch order."""

    def __init__(self, capacity: int):
        self.capacity = int(capacity)

    def start(self):
        _lib.check(_lib.load().mate_trace_start(self.capacity), "mate_trace_start")
        return self

    def stop(self):
        _lib.check(_lib.load().mate_trace_stop(), "mate_trace_stop")

    def read(self):
        lib = _lib.load()
        recs = (_lib.CTraceRecord * max(self.capacity, 1))()
        n = lib.mate_trace_read(recs, self.capacity)
        if n < 0:
            raise _lib.MateError(_lib.MATE_ERR_CUDA, "mate_trace_read")
        return [(lib.mate_kernel_name(recs[r].kernel).decode(), float(recs[r].ms)) for r in range(n)]


LOCALITY_MAPS = ("rms_order0", "rms_order1", "rms_order2", "rms_order3", "zigzag", "hilbert", "rms_rotation")


def scan_locality(T: int, H: int, W: int, kind: int, stream=None):
    """(sum of sequence distances, number of grid-adjacent pairs, largest distance) of index map `kind`
    over a T x H x W grid, computed on the GPU (see mate_scan_locality)."""
    out = torch.zeros(3, dtype=torch.int64, device="cuda")
    _lib.check(_lib.load().mate_scan_locality(int(T), int(H), int(W), int(kind), _p(out), _s(stream)),
               "mate_scan_locality")
    s, n, m = (int(v) for v in out.cpu().tolist())
    return s, n, m
