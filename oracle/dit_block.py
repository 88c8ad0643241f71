"""Plain fp64 CPU oracle of a DiT block with the MATE block as its token mixer.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may import this module.  It shares no code with the CUDA library and imports nothing from it.

The pages say MATE replaces the self-attention of a DiT and leaves the rest of the block unchanged ([ABS];
[NEWS] method), without describing that rest.  This module takes the standard DiT block with adaLN-Zero
conditioning as that plainest reading:
  * d-1  a conditioning vector c (timestep and pooled text embedding, per sample) gives six modulation
         vectors: [shift_a, scale_a, gate_a, shift_m, scale_m, gate_m] = silu(c) W_ada^T + b_ada;
  * d-2  layer norms without affine parameters, eps = 1e-6, over the channel dimension;
  * d-3  X1 = X + gate_a * MATE(LN(X) * (1 + scale_a) + shift_a)   (the token mixer: mate_oracle's block);
  * d-4  X2 = X1 + gate_m * MLP(LN(X1) * (1 + scale_m) + shift_m), MLP = W2 gelu_tanh(W1 h + b1) + b2 with
         hidden width 4 d;
  * d-5  no cross-attention (the pages do not mention one; text conditioning enters through c).
"""
from __future__ import annotations

import math

import numpy as np

from .mate_oracle import mate_forward

LN_EPS = 1e-6


def layer_norm(x: np.ndarray, eps: float = LN_EPS) -> np.ndarray:
    """Each row of x normalised to zero mean and unit variance (population variance, eps inside the root)."""
    x = np.asarray(x, np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def gelu_tanh(v: np.ndarray) -> np.ndarray:
    """GELU in its tanh form: v/2 (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3)))."""
    v = np.asarray(v, np.float64)
    return 0.5 * v * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (v + 0.044715 * v ** 3)))


def silu(v: np.ndarray) -> np.ndarray:
    v = np.asarray(v, np.float64)
    return v * 0.5 * (1.0 + np.tanh(0.5 * v))


def modulation(c: np.ndarray, w: dict) -> list:
    """The six modulation vectors [shift_a, scale_a, gate_a, shift_m, scale_m, gate_m] of one sample."""
    mod = silu(c) @ np.asarray(w["W_ada"], np.float64).T + np.asarray(w["b_ada"], np.float64)
    return np.split(mod, 6)


def mlp(h: np.ndarray, w: dict) -> np.ndarray:
    z = h @ np.asarray(w["W1"], np.float64).T + np.asarray(w["b1"], np.float64)
    return gelu_tanh(z) @ np.asarray(w["W2"], np.float64).T + np.asarray(w["b2"], np.float64)


def dit_block(X: np.ndarray, c: np.ndarray, w: dict, cfg, layer_idx: int) -> np.ndarray:
    """One DiT block with MATE as token mixer.  X [B, T, H, W, d], c [B, dc]; w holds the MATE weights plus
    W_ada [6d, dc], b_ada [6d], W1 [4d, d], b1 [4d], W2 [d, 4d], b2 [d]."""
    X = np.asarray(X, np.float64)
    Bn, T, H, W, d = X.shape
    out = np.empty_like(X)
    for b in range(Bn):
        sa, ca, ga, sm, cm, gm = modulation(np.asarray(c[b], np.float64), w)
        Xf = X[b].reshape(-1, d)
        h = layer_norm(Xf) * (1.0 + ca) + sa
        mix = mate_forward(h.reshape(1, T, H, W, d), w, cfg, layer_idx)[0].reshape(-1, d)
        X1 = Xf + ga * mix
        h2 = layer_norm(X1) * (1.0 + cm) + sm
        out[b] = (X1 + gm * mlp(h2, w)).reshape(T, H, W, d)
    return out
