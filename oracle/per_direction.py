"""Plain fp64 CPU oracle of the bidirectional scan and MATE block with separate parameters for the
backward scan direction.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may import this module.  It shares no code with the CUDA library and imports nothing from it.

The pages name a bidirectional Mamba2 block ([ABS]; [NEWS] method) without saying whether the two
directions share parameters.  The block oracle (mate_oracle) reads them as shared.  This module is the
other plain reading, kept as an option: the backward scan has its own A_log, D and dt_bias (same
in-projection, same B/C/x), y = y_forward + (y_backward reversed back).  Every step is a call of the
pinned single-direction recurrence; with the backward parameters equal to the forward ones it is the
shared-parameter oracle.
"""
from __future__ import annotations

import numpy as np

from .mate_oracle import _layer, in_projection, review_tokens, rms_permute, rms_unpermute, ssd_recurrence, te_branch


def ssd_bidirectional_per_direction(x, Bm, Cm, delta_f, A_f, D_f, delta_b, A_b, D_b, R: int) -> np.ndarray:
    """As mate_oracle.ssd_bidirectional, with (delta_b, A_b, D_b) for the scan over [prefix; video reversed]."""
    y_f = ssd_recurrence(x, Bm, Cm, delta_f, A_f, D_f)
    flip = np.concatenate([np.arange(R), np.arange(x.shape[0] - 1, R - 1, -1)])
    y_b = ssd_recurrence(x[flip], Bm[flip], Cm[flip], np.asarray(delta_b)[flip], A_b, D_b)
    return y_f[R:] + y_b[R:][::-1]


def ma_branch_per_direction(X3: np.ndarray, w: dict, cfg, layer_idx: int) -> np.ndarray:
    """MA branch for one sample with w['dt_bias_b'], w['A_log_b'], w['D_b'] for the backward scan."""
    order, _ = _layer(layer_idx)
    T, H, W, d = X3.shape
    Xp = rms_permute(np.asarray(X3, np.float64), order)
    Rv = review_tokens(X3, cfg.R, order)
    S = np.concatenate([Rv, Xp], axis=0)
    x, Bm, Cm, delta_f = in_projection(S, w, cfg)
    _, _, _, delta_b = in_projection(S, dict(w, dt_bias=w["dt_bias_b"]), cfg)
    A_f = -np.exp(np.asarray(w["A_log"], np.float64))
    A_b = -np.exp(np.asarray(w["A_log_b"], np.float64))
    y = ssd_bidirectional_per_direction(x, Bm, Cm, delta_f, A_f, w["D"], delta_b, A_b, w["D_b"], cfg.R)
    out_p = y.reshape(T * H * W, cfg.nh * cfg.P) @ np.asarray(w["W_out"], np.float64).T
    return rms_unpermute(out_p, order, T, H, W)


def mate_forward_per_direction(X: np.ndarray, w: dict, cfg, layer_idx: int) -> np.ndarray:
    """Out = MA + TE per sample, the MA branch with per-direction scan parameters."""
    X = np.asarray(X)
    return np.stack([ma_branch_per_direction(X[b], w, cfg, layer_idx) + te_branch(X[b], w, cfg, layer_idx)
                     for b in range(X.shape[0])])
