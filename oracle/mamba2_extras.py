"""Plain fp64 CPU oracle of the MATE block with the rest of the Mamba2 block around the scan: the short
causal depthwise convolution with SiLU on x, B and C, and the SiLU(z) gate with gated RMSNorm before the
out-projection.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may import this module.  It shares no code with the CUDA library and imports nothing from it.

The pages name the MA branch's core a (bidirectional) Mamba2 block ([ABS]; [NEWS] method) and say nothing
about its internals.  The block oracle (mate_oracle) keeps only the projections and the scan.  This module
adds the remaining parts of a Mamba2 block, read as follows:
  * e-1  a causal depthwise convolution of width 4 with a bias runs over the concatenated x | B | C
         channels of the in-projection, followed by SiLU; dt skips it (it only feeds the step size) and so
         does z;
  * e-2  the convolution runs once, along the sequence the forward scan reads ([review tokens; video rows
         in the layer's scan order]), zero-padded on the left of each sample; both scan directions read
         its output, so the bidirectional scan keeps one shared in-projection path;
  * e-3  the gate z is its own projection of the video rows, W_z [nh*P, d]; review rows need none (their
         outputs are dropped);
  * e-4  gated RMSNorm with the gate applied before the norm: g = y * silu(z), out = g / sqrt(mean(g^2) +
         eps) * norm_w over all nh*P channels of a row (one group), eps = 1e-5;
  * e-5  the out-projection reads the normalised rows.
Every other step is the pinned block oracle's.
"""
from __future__ import annotations

import numpy as np

from .mate_oracle import (_layer, in_projection, review_tokens, rms_permute, rms_unpermute, ssd_bidirectional,
                          te_branch)

CONV_K = 4          # width of the causal depthwise convolution
NORM_EPS = 1e-5     # epsilon of the gated RMSNorm


def silu(v: np.ndarray) -> np.ndarray:
    """SiLU(v) = v * sigmoid(v), with sigmoid written through tanh so that no exponential overflows."""
    v = np.asarray(v, np.float64)
    return v * 0.5 * (1.0 + np.tanh(0.5 * v))


def causal_conv(u: np.ndarray, w: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Depthwise causal convolution of the rows u [L, C]: out[t, c] = b[c] + sum_k w[c, k] u[t - K + 1 + k, c]
    with u = 0 before the first row (w [C, K], tap K - 1 on the current row)."""
    u = np.asarray(u, np.float64)
    w = np.asarray(w, np.float64)
    L, C = u.shape
    K = w.shape[1]
    padded = np.concatenate([np.zeros((K - 1, C)), u], axis=0)
    out = np.tile(np.asarray(b, np.float64), (L, 1))
    for k in range(K):
        out += w[:, k][None, :] * padded[k:k + L]
    return out


def gated_rmsnorm(y: np.ndarray, z: np.ndarray, weight: np.ndarray, eps: float = NORM_EPS) -> np.ndarray:
    """Rows of g = y * silu(z) scaled to unit root-mean-square (plus eps inside the root), times weight."""
    g = np.asarray(y, np.float64) * silu(z)
    return g / np.sqrt(np.mean(g * g, axis=-1, keepdims=True) + eps) * np.asarray(weight, np.float64)


def ma_branch_extras(X3: np.ndarray, w: dict, cfg, layer_idx: int) -> np.ndarray:
    """MA branch for one sample [T, H, W, d] with the convolution, the gate and the gated norm
    (w also holds W_z, conv_w [nh*P + 2N, 4], conv_b [nh*P + 2N], norm_w [nh*P])."""
    order, _ = _layer(layer_idx)
    T, H, W, d = X3.shape
    nP, N = cfg.nh * cfg.P, cfg.N
    Xp = rms_permute(np.asarray(X3, np.float64), order)
    Rv = review_tokens(X3, cfg.R, order)
    S = np.concatenate([Rv, Xp], axis=0)
    x, Bm, Cm, delta = in_projection(S, w, cfg)
    xbc = np.concatenate([x.reshape(-1, nP), Bm, Cm], axis=1)
    xbc = silu(causal_conv(xbc, w["conv_w"], w["conv_b"]))
    x = xbc[:, :nP].reshape(-1, cfg.nh, cfg.P)
    Bm, Cm = xbc[:, nP:nP + N], xbc[:, nP + N:]
    A = -np.exp(np.asarray(w["A_log"], np.float64))
    y = ssd_bidirectional(x, Bm, Cm, delta, A, w["D"], cfg.R).reshape(T * H * W, nP)
    z = Xp @ np.asarray(w["W_z"], np.float64).T
    out_p = gated_rmsnorm(y, z, w["norm_w"]) @ np.asarray(w["W_out"], np.float64).T
    return rms_unpermute(out_p, order, T, H, W)


def mate_forward_extras(X: np.ndarray, w: dict, cfg, layer_idx: int) -> np.ndarray:
    """Out = MA + TE per sample, the MA branch with the full Mamba2 block around the scan."""
    X = np.asarray(X)
    return np.stack([ma_branch_extras(X[b], w, cfg, layer_idx) + te_branch(X[b], w, cfg, layer_idx)
                     for b in range(X.shape[0])])
