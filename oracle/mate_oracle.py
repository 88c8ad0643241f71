"""Plain, slow, fp64 CPU oracle of the LinGen MATE block forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may import this module.  It shares no code with the CUDA library and imports nothing from it.

Sources (the pages describing the method):
  [NEWS]  LinGen news article ("视频生成模型太贵太慢怎么办", weiba1314 / xihudo), section
          "方法：线性复杂度的 MATE 模块" (method: the linear-complexity MATE block).
  [ABS]   "Towards High-Resolution Minute-Length Text-to-Video Generation with Linear Computational
          Complexity", abstract (English original).
  [FEAT]  "LinGen：基于Mamba机制的线性复杂度高清长视频生成框架", section "技术细节 / 关键算法创新"
          (Rotary Major Scan; TEmporal Swin Attention).

What the block computes ([ABS]; [NEWS] method): Out = MA(X) + TE(X), where
  MA = Rotary-Major-Scan reorder -> review tokens prepended -> bidirectional Mamba2 (SSD) scan between an
       in-projection and an out-projection -> reorder back;
  TE = TEmporal Swin Attention: attention inside small fixed 3D windows that shift on alternate layers.

Readings taken where the pages are silent (each is also listed in the design notes):
  * "1st priority" in unrolling = fastest-varying index ([NEWS] RMS paragraph, [FEAT] RMS list).
  * the four orders, fastest first: spatial-row (W,H,T), spatial-col (H,W,T), temporal-row (T,W,H),
    temporal-col (T,H,W); layer l uses order l mod 4.
  * bidirectional = same parameters both ways, outputs summed; review tokens prefixed in both directions
    in the same order, their outputs discarded.
  * review tokens = 3D average pool of X onto an (R/16) x 4 x 4 grid, ordered by the layer's scan order.
  * Mamba2 core: one B/C group, expand 1, A = -exp(A_log), delta = softplus(dt + dt_bias), zero initial
    state; recurrence h_t = exp(delta_t A) h_{t-1} + delta_t x_t B_t^T, y_t = h_t C_t + D x_t.
  * TESA: cyclic shift by minus the half window on odd layers, Swin region mask, scale 1/sqrt(tp), no
    biases; window and shift sizes from the block configuration.

Pins: every function here is checked by tests/test_oracle_pins.py against closed forms, brute force,
textbook reshapes and hand-derived fixtures (tests/golden/).  The composed block (mate_forward) is pinned
as a whole by a per-token closed form (every step forgetting its state, one-token attention windows: the
block reduces to [2 (delta (B . C) + D) x] W_out^T + v W_o^T on every scan order, review prefix included)
and by the sum-of-branches identity; the pages print no worked example of the block.
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np

# ----------------------------------------------------------------------------------------------------
# Rotary Major Scan ([NEWS] method, RMS paragraphs; [FEAT] 关键算法创新 / Rotary Major Scan)
# ----------------------------------------------------------------------------------------------------

# Axis priorities of the four scan orders, first priority (fastest-varying) first.
SCAN_ORDERS = {
    0: ("W", "H", "T"),  # spatial row-major: W first
    1: ("H", "W", "T"),  # spatial column-major: H first
    2: ("T", "W", "H"),  # temporal row-major: T first, then W
    3: ("T", "H", "W"),  # temporal column-major: T first, then H
}


def scan_positions(T: int, H: int, W: int, order: int) -> np.ndarray:
    """Position in the scanned sequence of every grid token (t, h, w), as an int64 array [T, H, W].

    Unrolls the grid with the order's first-priority axis innermost: nested loops from the last priority
    (outermost) to the first (innermost), a counter incrementing at every visit."""
    sizes = {"T": T, "H": H, "W": W}
    first, second, third = SCAN_ORDERS[order]
    pos = np.empty((T, H, W), dtype=np.int64)
    counter = 0
    idx = {"T": 0, "H": 0, "W": 0}
    for a in range(sizes[third]):
        idx[third] = a
        for b in range(sizes[second]):
            idx[second] = b
            for c in range(sizes[first]):
                idx[first] = c
                pos[idx["T"], idx["H"], idx["W"]] = counter
                counter += 1
    return pos


def rms_permute(X3: np.ndarray, order: int) -> np.ndarray:
    """Reorder a [T, H, W, d] grid into the scanned sequence [T*H*W, d]: row scan_positions[t,h,w] = X[t,h,w]."""
    T, H, W, d = X3.shape
    pos = scan_positions(T, H, W, order)
    out = np.empty((T * H * W, d), dtype=X3.dtype)
    for t in range(T):
        for h in range(H):
            out[pos[t, h]] = X3[t, h]  # all w of one (t, h) at once
    return out


def rms_unpermute(Xp: np.ndarray, order: int, T: int, H: int, W: int) -> np.ndarray:
    """Inverse of rms_permute: grid token (t, h, w) takes sequence row scan_positions[t, h, w]."""
    pos = scan_positions(T, H, W, order)
    out = np.empty((T, H, W, Xp.shape[1]), dtype=Xp.dtype)
    for t in range(T):
        for h in range(H):
            out[t, h] = Xp[pos[t, h]]
    return out


# ----------------------------------------------------------------------------------------------------
# Review tokens ([NEWS] method, review-token paragraph: an overview of the video tensor written into the
# Mamba hidden state ahead of the video tokens)
# ----------------------------------------------------------------------------------------------------

def review_grid(T: int, H: int, W: int, R: int):
    """The pooled grid (Tr, 4, 4) and pool factors for R review tokens; R must be 16 * Tr with Tr | T."""
    if R % 16 != 0:
        raise ValueError("R must be a multiple of 16")
    Tr = R // 16
    if Tr == 0:
        return (0, 4, 4), (1, H // 4, W // 4)
    if T % Tr or H % 4 or W % 4:
        raise ValueError("pooled grid does not divide the latent grid")
    return (Tr, 4, 4), (T // Tr, H // 4, W // 4)


def review_tokens(X3: np.ndarray, R: int, order: int) -> np.ndarray:
    """R review tokens [R, d]: block means of X over the pool cells, ordered by the layer's scan order."""
    T, H, W, d = X3.shape
    (Tr, Hr, Wr), (ft, fh, fw) = review_grid(T, H, W, R)
    if R == 0:
        return np.zeros((0, d), dtype=np.float64)
    pooled = np.zeros((Tr, Hr, Wr, d), dtype=np.float64)
    for a in range(Tr):
        for b in range(Hr):
            for c in range(Wr):
                cell = X3[a * ft:(a + 1) * ft, b * fh:(b + 1) * fh, c * fw:(c + 1) * fw, :]
                pooled[a, b, c] = cell.reshape(-1, d).astype(np.float64).sum(axis=0) / (ft * fh * fw)
    return rms_permute(pooled, order)


# ----------------------------------------------------------------------------------------------------
# Mamba2 selective scan ([ABS]: "bidirectional Mamba2 block"; [NEWS] method: Mamba2 is an SSM variant)
# ----------------------------------------------------------------------------------------------------

def softplus(v: np.ndarray) -> np.ndarray:
    """log(1 + e^v), evaluated without overflow."""
    v = np.asarray(v, dtype=np.float64)
    return np.where(v > 30.0, v, np.log1p(np.exp(np.minimum(v, 30.0))))


def ssd_recurrence(x: np.ndarray, Bm: np.ndarray, Cm: np.ndarray, delta: np.ndarray, A: np.ndarray,
                   D: np.ndarray, counter: Optional[Dict[str, int]] = None) -> np.ndarray:
    """The sequential per-token state-space recurrence, one state [P, N] per head, zero initial state:

        h_t = exp(delta_t * A) * h_{t-1} + delta_t * x_t B_t^T
        y_t = h_t C_t + D * x_t

    x [L, nh, P]; Bm, Cm [L, N] (one group shared by all heads); delta [L, nh]; A, D [nh].  Returns y [L, nh, P]."""
    x = np.asarray(x, np.float64)
    Bm = np.asarray(Bm, np.float64)
    Cm = np.asarray(Cm, np.float64)
    delta = np.asarray(delta, np.float64)
    A = np.asarray(A, np.float64)
    D = np.asarray(D, np.float64)
    L, nh, P = x.shape
    N = Bm.shape[1]
    h = np.zeros((nh, P, N))
    y = np.empty((L, nh, P))
    for t in range(L):
        decay = np.exp(delta[t] * A)                       # [nh]
        h = decay[:, None, None] * h + (delta[t][:, None] * x[t])[:, :, None] * Bm[t][None, None, :]
        y[t] = h @ Cm[t] + D[:, None] * x[t]
    if counter is not None:
        counter["ssd"] = counter.get("ssd", 0) + L * nh * P * N * 2
    return y


def ssd_bidirectional(x: np.ndarray, Bm: np.ndarray, Cm: np.ndarray, delta: np.ndarray, A: np.ndarray,
                      D: np.ndarray, R: int, counter: Optional[Dict[str, int]] = None) -> np.ndarray:
    """Bidirectional scan over S = [prefix (R rows); video rows].  The forward scan runs over S; the second
    scan runs over [prefix; video reversed], with the same parameters.  The prefix outputs are dropped and
    the video outputs summed (the second scan's reversed back).  Inputs are per-row arrays of S; returns
    [L - R, nh, P]."""
    y_f = ssd_recurrence(x, Bm, Cm, delta, A, D, counter)
    flip = np.concatenate([np.arange(R), np.arange(x.shape[0] - 1, R - 1, -1)])
    y_b = ssd_recurrence(x[flip], Bm[flip], Cm[flip], delta[flip], A, D, counter)
    return y_f[R:] + y_b[R:][::-1]


# ----------------------------------------------------------------------------------------------------
# TEmporal Swin Attention ([NEWS] method TESA paragraph; [FEAT] 关键算法创新 / TESA: small fixed 3D
# windows, window partition shifted between adjacent layers, linear in the token count)
# ----------------------------------------------------------------------------------------------------

def _region(p: int, D: int, w: int, s: int) -> int:
    """Swin region of shifted coordinate p on an axis of length D with window w and shift s."""
    if p < D - w:
        return 0
    if p < D - s:
        return 1
    return 2


def tesa_attention(qkv: np.ndarray, th: int, tp: int, window, shift, shifted: bool,
                   counter: Optional[Dict[str, int]] = None) -> np.ndarray:
    """Window attention on a [T, H, W, 3*th*tp] grid of q | k | v (head-major).  Returns [T, H, W, th*tp].

    Unshifted layers partition the grid into (wt, wh, ww) windows.  Shifted layers first roll the grid by
    minus the shift on every axis (shifted position p holds original token (p + s) mod D), partition that,
    and forbid attention between tokens of different wrap regions; the result is rolled back.  Inside a
    window each query attends to the allowed keys with softmax(q.k / sqrt(tp))."""
    T, H, W, _ = qkv.shape
    wt, wh, ww = window
    st, sh, sw = shift if shifted else (0, 0, 0)
    if T % wt or H % wh or W % ww:
        raise ValueError("window must divide the grid")
    q = np.asarray(qkv[..., 0 * th * tp:1 * th * tp], np.float64).reshape(T, H, W, th, tp)
    k = np.asarray(qkv[..., 1 * th * tp:2 * th * tp], np.float64).reshape(T, H, W, th, tp)
    v = np.asarray(qkv[..., 2 * th * tp:3 * th * tp], np.float64).reshape(T, H, W, th, tp)
    out = np.zeros((T, H, W, th, tp))
    scale = 1.0 / math.sqrt(tp)
    for a in range(T // wt):
        for b in range(H // wh):
            for c in range(W // ww):
                members = []   # original coordinates of the window's tokens
                regions = []
                for pt in range(a * wt, (a + 1) * wt):
                    for ph in range(b * wh, (b + 1) * wh):
                        for pw in range(c * ww, (c + 1) * ww):
                            members.append(((pt + st) % T, (ph + sh) % H, (pw + sw) % W))
                            if shifted:
                                regions.append((_region(pt, T, wt, st), _region(ph, H, wh, sh),
                                                _region(pw, W, ww, sw)))
                            else:
                                regions.append((0, 0, 0))
                it = np.array([m[0] for m in members])
                ih = np.array([m[1] for m in members])
                iw = np.array([m[2] for m in members])
                Qw, Kw, Vw = q[it, ih, iw], k[it, ih, iw], v[it, ih, iw]      # [m, th, tp]
                m = len(members)
                reg = np.array(regions)                                       # [m, 3]
                allowed = (reg[:, None, :] == reg[None, :, :]).all(axis=2)    # same region on every axis
                scores = np.einsum("ihc,jhc->hij", Qw, Kw) * scale
                scores = np.where(allowed[None], scores, -np.inf)
                scores = scores - scores.max(axis=2, keepdims=True)
                prob = np.exp(scores)
                prob = prob / prob.sum(axis=2, keepdims=True)
                out[it, ih, iw] = np.einsum("hij,jhc->ihc", prob, Vw)
                if counter is not None:
                    counter["tesa"] = counter.get("tesa", 0) + 2 * th * m * m * tp
    return out.reshape(T, H, W, th * tp)


# ----------------------------------------------------------------------------------------------------
# The MATE block ([ABS]; [NEWS] method: MATE = MA branch + TE branch, replacing DiT self-attention)
# ----------------------------------------------------------------------------------------------------

def _layer(layer_idx: int):
    return layer_idx % 4, layer_idx % 2 == 1


def in_projection(S: np.ndarray, w: dict, cfg, counter=None):
    """Split the MA in-projection of the rows S [L, d] into x [L, nh, P], B, C [L, N] and delta [L, nh]."""
    Z = np.asarray(S, np.float64) @ np.asarray(w["W_in"], np.float64).T
    if counter is not None:
        counter["proj"] = counter.get("proj", 0) + Z.shape[0] * Z.shape[1] * S.shape[1]
    nP = cfg.nh * cfg.P
    x = Z[:, :nP].reshape(-1, cfg.nh, cfg.P)
    Bm = Z[:, nP:nP + cfg.N]
    Cm = Z[:, nP + cfg.N:nP + 2 * cfg.N]
    dt = Z[:, nP + 2 * cfg.N:]
    delta = softplus(dt + np.asarray(w["dt_bias"], np.float64)[None, :])
    return x, Bm, Cm, delta


def ma_branch(X3: np.ndarray, w: dict, cfg, layer_idx: int, counter=None) -> np.ndarray:
    """MA branch for one sample [T, H, W, d] -> [T, H, W, d]."""
    order, _ = _layer(layer_idx)
    T, H, W, d = X3.shape
    Xp = rms_permute(np.asarray(X3, np.float64), order)
    Rv = review_tokens(X3, cfg.R, order)
    S = np.concatenate([Rv, Xp], axis=0)
    x, Bm, Cm, delta = in_projection(S, w, cfg, counter)
    A = -np.exp(np.asarray(w["A_log"], np.float64))
    y = ssd_bidirectional(x, Bm, Cm, delta, A, w["D"], cfg.R, counter)      # [n, nh, P]
    out_p = y.reshape(T * H * W, cfg.nh * cfg.P) @ np.asarray(w["W_out"], np.float64).T
    if counter is not None:
        counter["proj"] = counter.get("proj", 0) + out_p.shape[0] * out_p.shape[1] * cfg.nh * cfg.P
    return rms_unpermute(out_p, order, T, H, W)


def te_branch(X3: np.ndarray, w: dict, cfg, layer_idx: int, counter=None) -> np.ndarray:
    """TE branch for one sample: qkv projection, TESA, output projection."""
    _, shifted = _layer(layer_idx)
    T, H, W, d = X3.shape
    qkv = np.asarray(X3, np.float64).reshape(-1, d) @ np.asarray(w["W_qkv"], np.float64).T
    O = tesa_attention(qkv.reshape(T, H, W, -1), cfg.th, cfg.tp, (cfg.wt, cfg.wh, cfg.ww),
                       (cfg.st, cfg.sh, cfg.sw), shifted, counter)
    out = O.reshape(-1, cfg.th * cfg.tp) @ np.asarray(w["W_o"], np.float64).T
    if counter is not None:
        counter["proj"] = counter.get("proj", 0) + qkv.shape[0] * qkv.shape[1] * d + out.shape[0] * d * O.shape[-1]
    return out.reshape(T, H, W, d)


def mate_forward(X: np.ndarray, w: dict, cfg, layer_idx: int, counter=None) -> np.ndarray:
    """The MATE block: Out = MA(X) + TE(X) for X [B, T, H, W, d]; both branches read the same X."""
    return np.stack([ma_branch(X[b], w, cfg, layer_idx, counter) + te_branch(X[b], w, cfg, layer_idx, counter)
                     for b in range(X.shape[0])])
