"""Seeded synthetic inputs and weights for the MATE block (shared by the oracle and the CUDA path).

This module holds no arithmetic of the method itself: it only names the block's shapes and draws the
random tensors both sides consume, so that the oracle and the GPU path see identical bits.

Shapes follow the LinGen MATE block ("Towards High-Resolution Minute-Length Text-to-Video Generation
with Linear Computational Complexity", abstract; MATE = MA branch + TE branch):

* latent token grid X: [B, T, H, W, d] channels-last;
* MA in-projection W_in: [nh*P + 2*N + nh, d] (out_features x in_features), output features ordered
  x (head-major, head h at [h*P, (h+1)*P)) | B (N) | C (N) | dt (nh);
* dt_bias, A_log, D: [nh];
* MA out-projection W_out: [d, nh*P];
* TE projections W_qkv: [3*th*tp, d] ordered q | k | v, head-major inside each; W_o: [d, th*tp].

Draw order (one numpy PCG64 stream per seed): X, W_in, A_log, D, W_out, W_qkv, W_o.  dt_bias is zero
unless overridden.  Linear weights are N(0,1)/sqrt(fan_in), A_log ~ U[0,1], D ~ N(0,1), X ~ N(0,1).
For bf16 configurations every tensor is rounded to bf16 (round-to-nearest-even) once, after drawing.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class MateConfig:
    """Shape of one MATE block.  Window (wt, wh, ww); Swin shift (st, sh, sw) is applied on odd layers."""

    name: str
    B: int
    T: int
    H: int
    W: int
    d: int
    nh: int
    P: int
    N: int
    Q: int
    R: int
    th: int
    tp: int
    wt: int
    wh: int
    ww: int
    st: int
    sh: int
    sw: int
    dtype: str  # "bf16" or "f32"
    seed: int

    @property
    def n(self) -> int:
        return self.T * self.H * self.W

    @property
    def L(self) -> int:
        return self.R + self.n

    @property
    def d_inner(self) -> int:
        return self.nh * self.P

    @property
    def d_in_proj(self) -> int:
        return self.nh * self.P + 2 * self.N + self.nh

    @property
    def d_attn(self) -> int:
        return self.th * self.tp


def _cfg(name, B, T, H, W, d, nh, P, N, Q, R, th, tp, win, dtype, seed, shift=None):
    wt, wh, ww = win
    st, sh, sw = shift if shift is not None else (wt // 2, wh // 2, ww // 2)
    return MateConfig(name, B, T, H, W, d, nh, P, N, Q, R, th, tp, wt, wh, ww, st, sh, sw, dtype, seed)


# The five workloads of the block: a tiny fp32 case, then bf16 latent grids of 16k, 65k and 262k
# tokens at d_model 1024, and a 2 x 147k-token grid at d_model 2048.
CONFIGS: Dict[str, MateConfig] = {
    "tiny_f32_4x8x8": _cfg("tiny_f32_4x8x8", 1, 4, 8, 8, 64, 2, 32, 16, 64, 16, 2, 32, (2, 4, 4), "f32", 0,
                           shift=(1, 2, 2)),
    "bf16_16x32x32": _cfg("bf16_16x32x32", 1, 16, 32, 32, 1024, 16, 64, 128, 256, 256, 8, 128, (4, 8, 8),
                          "bf16", 1),
    "bf16_64x32x32": _cfg("bf16_64x32x32", 1, 64, 32, 32, 1024, 16, 64, 128, 256, 256, 8, 128, (4, 8, 8),
                          "bf16", 2),
    "bf16_256x32x32": _cfg("bf16_256x32x32", 1, 256, 32, 32, 1024, 16, 64, 128, 256, 1024, 8, 128, (4, 8, 8),
                           "bf16", 3),
    "bf16_2x64x48x48_d2048": _cfg("bf16_2x64x48x48_d2048", 2, 64, 48, 48, 2048, 32, 64, 128, 256, 512, 16, 128,
                                  (4, 8, 8), "bf16", 4),
}

# Smaller bf16 shapes with the production head/state/window sizes, for parity tests the oracle finishes
# in seconds.  They span several GEMM tiles, SSD chunks and windows, and some have ragged review chunks
# (R not a multiple of Q) and partial GEMM row tiles.
TEST_CONFIGS: Dict[str, MateConfig] = {
    "bf16_small_8x16x16": _cfg("bf16_small_8x16x16", 1, 8, 16, 16, 1024, 16, 64, 128, 256, 128, 8, 128, (4, 8, 8),
                               "bf16", 11),
    "bf16_ragged_12x16x24": _cfg("bf16_ragged_12x16x24", 1, 12, 16, 24, 1024, 16, 64, 128, 256, 48, 8, 128,
                                 (4, 8, 8), "bf16", 12),
    "bf16_b2_20x16x16_d512": _cfg("bf16_b2_20x16x16_d512", 2, 20, 16, 16, 512, 8, 64, 128, 256, 320, 4, 128,
                                  (4, 8, 8), "bf16", 13),
    "f32_b2_4x8x12": _cfg("f32_b2_4x8x12", 2, 4, 8, 12, 64, 2, 32, 16, 64, 32, 2, 32, (2, 4, 4), "f32", 14,
                          shift=(1, 2, 2)),
}


def all_configs() -> Dict[str, MateConfig]:
    out = dict(CONFIGS)
    out.update(TEST_CONFIGS)
    return out


def layer_schedule(layer_idx: int):
    """(scan order, shifted) used by layer `layer_idx`: orders cycle 0..3, the Swin shift alternates."""
    return layer_idx % 4, layer_idx % 2 == 1


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bf16 (ties to even); returned as float32 holding bf16 values."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = ((u.astype(np.uint64) + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32)
    return (r << 16).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The upper 16 bits of float32 values that are already bf16-representable."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    return (u >> 16).astype(np.uint16)


def make_inputs(cfg: MateConfig, seed: Optional[int] = None, *, dt_bias: Optional[float] = None,
                a_log_range=(0.0, 1.0), x_scale: float = 1.0) -> Dict[str, np.ndarray]:
    """Draw X and the block's weights for `cfg`.  Values are float32 (bf16-representable for bf16 configs).

    `dt_bias` (a constant) and `a_log_range` override the default initialisation; a negative dt_bias
    (small step sizes) together with a low A_log range gives the scan a long memory, which exercises the
    inter-chunk state carry."""
    rng = np.random.default_rng(cfg.seed if seed is None else seed)
    f32 = np.float32

    def lin(out_f, in_f):
        return (rng.standard_normal((out_f, in_f)) / np.sqrt(in_f)).astype(f32)

    X = (rng.standard_normal((cfg.B, cfg.T, cfg.H, cfg.W, cfg.d)) * x_scale).astype(f32)
    W_in = lin(cfg.d_in_proj, cfg.d)
    A_log = rng.uniform(a_log_range[0], a_log_range[1], size=cfg.nh).astype(f32)
    D = rng.standard_normal(cfg.nh).astype(f32)
    W_out = lin(cfg.d, cfg.d_inner)
    W_qkv = lin(3 * cfg.d_attn, cfg.d)
    W_o = lin(cfg.d, cfg.d_attn)
    dtb = np.full(cfg.nh, 0.0 if dt_bias is None else dt_bias, dtype=f32)
    out = dict(X=X, W_in=W_in, dt_bias=dtb, A_log=A_log, D=D, W_out=W_out, W_qkv=W_qkv, W_o=W_o)
    if cfg.dtype == "bf16":
        # Large tensors (X, projection weights) are stored in bf16; the per-head scalars stay fp32.
        for k in ("X", "W_in", "W_out", "W_qkv", "W_o"):
            out[k] = round_to_bf16(out[k])
    return out


def make_x_only(cfg: MateConfig, seed: int) -> np.ndarray:
    """A fresh latent grid X with the config's shape (bf16-rounded for bf16 configs)."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((cfg.B, cfg.T, cfg.H, cfg.W, cfg.d)).astype(np.float32)
    return round_to_bf16(X) if cfg.dtype == "bf16" else X
