"""Plain fp64 CPU oracle of the MATE block's backward pass: the gradients of the bidirectional selective
scan, of TEmporal Swin Attention and of the whole block with respect to its input and weights.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may import this module.  It shares no code with the CUDA library and imports nothing from it.

The pages describe only the forward computation ([ABS]; [NEWS] method); training the block needs its
gradients, which follow from the forward definitions by the chain rule.  Each function here is the
adjoint of the forward oracle function it names, written out step by step in reverse order:
  * the recurrence h_t = a_t h_{t-1} + delta_t x_t B_t^T, y_t = h_t C_t + D x_t with a_t = exp(delta_t A)
    has the adjoint state G_t = dy_t C_t^T + a_{t+1} G_{t+1} (run from the last row to the first), and
        dx_t = delta_t G_t B_t + D dy_t            dB_t = delta_t G_t^T x_t      dC_t = h_t^T dy_t
        ddelta_t = x_t^T G_t B_t + A a_t <h_{t-1}, G_t>       dA = sum_t delta_t a_t <h_{t-1}, G_t>
        dD = sum_t <x_t, dy_t>                      (B and C gradients summed over heads);
  * the bidirectional scan feeds the video rows' output gradient to both directions (the second one in
    its flipped order) and maps the second direction's input gradients back through the flip;
  * window attention: dV = P^T dO, dP = dO V^T, dS = P (dP - rowsum(dP P)), dQ = dS K / sqrt(tp),
    dK = dS^T Q / sqrt(tp), masked pairs carrying no gradient;
  * permutations (the scan orders) have their inverse as adjoint; the review pooling spreads each review
    token's gradient evenly over its pool cell; linear maps transpose.
Pinned against central finite differences of the forward oracle.
"""
from __future__ import annotations

import math

import numpy as np

from .mate_oracle import (_layer, _region, in_projection, review_grid, review_tokens, rms_permute,
                          rms_unpermute, ssd_bidirectional, tesa_attention)


def ssd_recurrence_backward(x, Bm, Cm, delta, A, D, dy):
    """Gradients of mate_oracle.ssd_recurrence's output y with respect to its inputs, given dy [L, nh, P].
    Returns dx [L, nh, P], dB [L, N], dC [L, N], ddelta [L, nh], dA [nh], dD [nh]."""
    x, Bm, Cm, delta, A, D, dy = (np.asarray(v, np.float64) for v in (x, Bm, Cm, delta, A, D, dy))
    L, nh, P = x.shape
    N = Bm.shape[1]
    # forward pass, keeping every state: hs[t + 1] = h_t, hs[0] = 0
    a = np.exp(delta * A[None, :])                                     # [L, nh]
    hs = np.zeros((L + 1, nh, P, N))
    for t in range(L):
        hs[t + 1] = a[t][:, None, None] * hs[t] + (delta[t][:, None] * x[t])[:, :, None] * Bm[t][None, None, :]
    dx, dB, dC = np.zeros_like(x), np.zeros_like(Bm), np.zeros_like(Cm)
    ddelta, dA, dD = np.zeros_like(delta), np.zeros(nh), np.zeros(nh)
    G = np.zeros((nh, P, N))
    for t in range(L - 1, -1, -1):
        if t + 1 < L:
            G = a[t + 1][:, None, None] * G
        else:
            G = np.zeros((nh, P, N))
        G = G + dy[t][:, :, None] * Cm[t][None, None, :]
        dC[t] = np.einsum("hpn,hp->n", hs[t + 1], dy[t])
        dx[t] = delta[t][:, None] * np.einsum("hpn,n->hp", G, Bm[t]) + D[:, None] * dy[t]
        dB[t] = np.einsum("hpn,hp->n", G, delta[t][:, None] * x[t])
        hg = np.einsum("hpn,hpn->h", hs[t], G)                        # <h_{t-1}, G_t> per head
        ddelta[t] = np.einsum("hp,hpn,n->h", x[t], G, Bm[t]) + A * a[t] * hg
        dA += delta[t] * a[t] * hg
        dD += np.einsum("hp,hp->h", x[t], dy[t])
    return dx, dB, dC, ddelta, dA, dD


def ssd_bidirectional_backward(x, Bm, Cm, delta, A, D, R: int, dy):
    """Gradients of mate_oracle.ssd_bidirectional (prefix R rows, video output gradient dy [L - R, nh, P])
    with respect to x, Bm, Cm, delta (all rows of S), A and D."""
    x = np.asarray(x, np.float64)
    L, nh, P = x.shape
    dy = np.asarray(dy, np.float64)
    dyf = np.zeros((L, nh, P))
    dyf[R:] = dy
    gf = ssd_recurrence_backward(x, Bm, Cm, delta, A, D, dyf)
    flip = np.concatenate([np.arange(R), np.arange(L - 1, R - 1, -1)])
    dyb = np.zeros((L, nh, P))
    dyb[R:] = dy[::-1]
    Bm, Cm, delta = (np.asarray(v, np.float64) for v in (Bm, Cm, delta))
    gb = ssd_recurrence_backward(x[flip], Bm[flip], Cm[flip], delta[flip], A, D, dyb)
    out = []
    for f, b in zip(gf[:4], gb[:4]):     # per-row gradients: the second direction's rows sit at flip
        g = f.copy()
        g[flip] += b
        out.append(g)
    return out[0], out[1], out[2], out[3], gf[4] + gb[4], gf[5] + gb[5]


def tesa_attention_backward(qkv, th: int, tp: int, window, shift, shifted: bool, dO):
    """Gradient of mate_oracle.tesa_attention's output [T, H, W, th*tp] with respect to its q | k | v input,
    given dO of the output's shape.  Returns dqkv [T, H, W, 3*th*tp]."""
    T, H, W, _ = qkv.shape
    wt, wh, ww = window
    st, sh, sw = shift if shifted else (0, 0, 0)
    q = np.asarray(qkv[..., 0 * th * tp:1 * th * tp], np.float64).reshape(T, H, W, th, tp)
    k = np.asarray(qkv[..., 1 * th * tp:2 * th * tp], np.float64).reshape(T, H, W, th, tp)
    v = np.asarray(qkv[..., 2 * th * tp:3 * th * tp], np.float64).reshape(T, H, W, th, tp)
    dO = np.asarray(dO, np.float64).reshape(T, H, W, th, tp)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    scale = 1.0 / math.sqrt(tp)
    for a_ in range(T // wt):
        for b_ in range(H // wh):
            for c_ in range(W // ww):
                members, regions = [], []
                for pt in range(a_ * wt, (a_ + 1) * wt):
                    for ph in range(b_ * wh, (b_ + 1) * wh):
                        for pw in range(c_ * ww, (c_ + 1) * ww):
                            members.append(((pt + st) % T, (ph + sh) % H, (pw + sw) % W))
                            regions.append((_region(pt, T, wt, st), _region(ph, H, wh, sh), _region(pw, W, ww, sw))
                                           if shifted else (0, 0, 0))
                it = np.array([m[0] for m in members])
                ih = np.array([m[1] for m in members])
                iw = np.array([m[2] for m in members])
                Qw, Kw, Vw, dOw = q[it, ih, iw], k[it, ih, iw], v[it, ih, iw], dO[it, ih, iw]
                reg = np.array(regions)
                allowed = (reg[:, None, :] == reg[None, :, :]).all(axis=2)
                scores = np.einsum("ihc,jhc->hij", Qw, Kw) * scale
                scores = np.where(allowed[None], scores, -np.inf)
                scores = scores - scores.max(axis=2, keepdims=True)
                prob = np.exp(scores)
                prob = prob / prob.sum(axis=2, keepdims=True)            # [th, m, m]
                dV = np.einsum("hij,ihc->jhc", prob, dOw)
                dP = np.einsum("ihc,jhc->hij", dOw, Vw)
                dS = prob * (dP - (dP * prob).sum(axis=2, keepdims=True))
                dq[it, ih, iw] += scale * np.einsum("hij,jhc->ihc", dS, Kw)
                dk[it, ih, iw] += scale * np.einsum("hij,ihc->jhc", dS, Qw)
                dv[it, ih, iw] += dV
    return np.concatenate([dq.reshape(T, H, W, -1), dk.reshape(T, H, W, -1), dv.reshape(T, H, W, -1)], axis=-1)


def _review_tokens_backward(dRv, T: int, H: int, W: int, R: int, order: int):
    """Adjoint of mate_oracle.review_tokens: each pooled cell's gradient spread evenly over the cell."""
    d = dRv.shape[1]
    dX3 = np.zeros((T, H, W, d))
    if R == 0:
        return dX3
    (Tr, Hr, Wr), (ft, fh, fw) = review_grid(T, H, W, R)
    dpooled = rms_unpermute(np.asarray(dRv, np.float64), order, Tr, Hr, Wr)
    for a in range(Tr):
        for b in range(Hr):
            for c in range(Wr):
                dX3[a * ft:(a + 1) * ft, b * fh:(b + 1) * fh, c * fw:(c + 1) * fw, :] += \
                    dpooled[a, b, c] / (ft * fh * fw)
    return dX3


def ma_branch_backward(X3, w: dict, cfg, layer_idx: int, dMA):
    """Gradients of mate_oracle.ma_branch for one sample: (dX3, {W_in, dt_bias, A_log, D, W_out})."""
    order, _ = _layer(layer_idx)
    X3 = np.asarray(X3, np.float64)
    T, H, W, d = X3.shape
    nP, N, R = cfg.nh * cfg.P, cfg.N, cfg.R
    W_in, W_out = np.asarray(w["W_in"], np.float64), np.asarray(w["W_out"], np.float64)
    # forward, keeping what the backward pass reads
    Xp = rms_permute(X3, order)
    Rv = review_tokens(X3, R, order)
    S = np.concatenate([Rv, Xp], axis=0)
    x, Bm, Cm, delta = in_projection(S, w, cfg)
    Z = S @ W_in.T
    A = -np.exp(np.asarray(w["A_log"], np.float64))
    y = ssd_bidirectional(x, Bm, Cm, delta, A, w["D"], R).reshape(T * H * W, nP)
    # backward
    dout_p = rms_permute(np.asarray(dMA, np.float64), order)                   # adjoint of the unpermute
    dW_out = dout_p.T @ y
    dy = (dout_p @ W_out).reshape(T * H * W, cfg.nh, cfg.P)
    dx, dB, dC, ddelta, dA, dD = ssd_bidirectional_backward(x, Bm, Cm, delta, A, w["D"], R, dy)
    dt_raw = Z[:, nP + 2 * N:] + np.asarray(w["dt_bias"], np.float64)[None, :]
    ddt = ddelta * (1.0 / (1.0 + np.exp(-dt_raw)))                              # softplus' = sigmoid
    dZ = np.concatenate([dx.reshape(-1, nP), dB, dC, ddt], axis=1)
    dW_in = dZ.T @ S
    dS = dZ @ W_in
    dX3 = rms_unpermute(dS[R:], order, T, H, W) + _review_tokens_backward(dS[:R], T, H, W, R, order)
    grads = {"W_in": dW_in, "dt_bias": ddt.sum(axis=0), "A_log": dA * A, "D": dD, "W_out": dW_out}
    return dX3, grads


def te_branch_backward(X3, w: dict, cfg, layer_idx: int, dTE):
    """Gradients of mate_oracle.te_branch for one sample: (dX3, {W_qkv, W_o})."""
    _, shifted = _layer(layer_idx)
    X3 = np.asarray(X3, np.float64)
    T, H, W, d = X3.shape
    W_qkv, W_o = np.asarray(w["W_qkv"], np.float64), np.asarray(w["W_o"], np.float64)
    Xf = X3.reshape(-1, d)
    qkv = Xf @ W_qkv.T
    win, sh = (cfg.wt, cfg.wh, cfg.ww), (cfg.st, cfg.sh, cfg.sw)
    O = tesa_attention(qkv.reshape(T, H, W, -1), cfg.th, cfg.tp, win, sh, shifted).reshape(-1, cfg.th * cfg.tp)
    dTEf = np.asarray(dTE, np.float64).reshape(-1, d)
    dW_o = dTEf.T @ O
    dO = dTEf @ W_o
    dqkv = tesa_attention_backward(qkv.reshape(T, H, W, -1), cfg.th, cfg.tp, win, sh, shifted,
                                   dO.reshape(T, H, W, -1)).reshape(-1, 3 * cfg.th * cfg.tp)
    dW_qkv = dqkv.T @ Xf
    dX3 = (dqkv @ W_qkv).reshape(T, H, W, d)
    return dX3, {"W_qkv": dW_qkv, "W_o": dW_o}


def mate_backward(X, w: dict, cfg, layer_idx: int, dOut):
    """Gradients of mate_oracle.mate_forward: (dX [B, T, H, W, d], weight gradients summed over samples)."""
    X = np.asarray(X, np.float64)
    dOut = np.asarray(dOut, np.float64)
    dX = np.zeros_like(X)
    grads = {}
    for b in range(X.shape[0]):
        dxm, gm = ma_branch_backward(X[b], w, cfg, layer_idx, dOut[b])
        dxt, gt = te_branch_backward(X[b], w, cfg, layer_idx, dOut[b])
        dX[b] = dxm + dxt
        for k, v in {**gm, **gt}.items():
            grads[k] = grads.get(k, 0.0) + v
    return dX, grads


__all__ = ["ssd_recurrence_backward", "ssd_bidirectional_backward", "tesa_attention_backward",
           "ma_branch_backward", "te_branch_backward", "mate_backward"]
