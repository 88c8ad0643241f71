"""Error floor of bf16 storage for the MATE block, computed with the fp64 oracle.

A bf16 block keeps its tensors in bf16 between steps: the review tokens, the projected x / B / C / q / k / v,
the scan output y, the attention output O and the block output.  Rounding exactly those tensors (and
nothing else) inside the fp64 oracle gives the error that ANY bf16-storage implementation carries, even
one whose arithmetic is otherwise exact.  For this workload the block output is heavy-tailed (the MA
branch scales each token by its own C_i . B_i delta_i), so that floor, measured as max|err| / rms(out),
lies above 2e-2.  The tests therefore require the GPU's RMS-normalised error to stay within
max(2e-2, 1.5 x floor) next to the 2e-2 relative bound (see the design notes)."""
import numpy as np

import mate_inputs as mi
from oracle import mate_oracle as O

r16 = mi.round_to_bf16


def _r(a):
    return r16(np.asarray(a, np.float64)).astype(np.float64)


def bf16_storage_forward(X, w, cfg, layer):
    """The oracle's block with bf16 rounding applied at the storage points listed in the module docstring."""
    order, shifted = layer % 4, layer % 2 == 1
    outs = []
    for b in range(X.shape[0]):
        X3 = np.asarray(X[b], np.float64)
        T, H, W, d = X3.shape
        Xp = O.rms_permute(X3, order)
        Rv = _r(O.review_tokens(X3, cfg.R, order))
        S = np.concatenate([Rv, Xp], axis=0)
        x, Bm, Cm, delta = O.in_projection(S, w, cfg)
        x, Bm, Cm = _r(x), _r(Bm), _r(Cm)
        A = -np.exp(np.asarray(w["A_log"], np.float64))
        y = _r(O.ssd_bidirectional(x, Bm, Cm, delta, A, w["D"], cfg.R).reshape(T * H * W, -1))
        ma = O.rms_unpermute(y @ np.asarray(w["W_out"], np.float64).T, order, T, H, W)
        qkv = _r(X3.reshape(-1, d) @ np.asarray(w["W_qkv"], np.float64).T)
        Oa = _r(O.tesa_attention(qkv.reshape(T, H, W, -1), cfg.th, cfg.tp, (cfg.wt, cfg.wh, cfg.ww),
                                 (cfg.st, cfg.sh, cfg.sw), shifted))
        te = (Oa.reshape(-1, cfg.th * cfg.tp) @ np.asarray(w["W_o"], np.float64).T).reshape(T, H, W, d)
        outs.append(_r(ma + te))
    return np.stack(outs)


def rms_normalised_max_err(a, ref):
    ref = np.asarray(ref, np.float64)
    return float(np.abs(np.asarray(a, np.float64) - ref).max() / np.sqrt(np.mean(ref * ref)))


def ssd_bf16_storage_emulation(x, Bm, Cm, delta, A, D, R, Q=256):
    """Chunked bidirectional scan in exact (fp64) arithmetic that rounds to bf16 only what a bf16
    tensor-core scan must hold in bf16: the MMA operands (G = C B^T, the intra-chunk coefficients,
    the decay-weighted inputs of the chunk states, the carried states) and the stored chunk states and
    output.  The scan test bounds the GPU's element-wise error by this emulation's error (the GPU adds
    only accumulation-order differences on top).  x [L, nh, P], Bm / Cm [L, N], delta [L, nh]."""
    x, Bm, Cm, delta = (np.asarray(a, np.float64) for a in (x, Bm, Cm, delta))
    A, D = np.asarray(A, np.float64), np.asarray(D, np.float64)
    L, nh, P = x.shape
    N = Bm.shape[1]
    n = L - R
    nRc, nVc = -(-R // Q), -(-n // Q)
    chunks = [(c * Q, min(c * Q + Q, R)) for c in range(nRc)] + [(R + v * Q, R + min(v * Q + Q, n)) for v in range(nVc)]
    out = np.zeros((n, nh, P))
    for h in range(nh):
        Sf, Sb, gl = [], [], []
        for a0, a1 in chunks:
            a = delta[a0:a1, h] * A[h]
            s = np.cumsum(a)
            wf = np.exp(s[-1] - s) * delta[a0:a1, h]
            wb = np.exp(s - a) * delta[a0:a1, h]
            Sf.append(_r(_r(wf[:, None] * x[a0:a1, h]).T @ Bm[a0:a1]))
            Sb.append(_r(_r(wb[:, None] * x[a0:a1, h]).T @ Bm[a0:a1]))
            gl.append(s[-1])
        H = np.zeros((P, N))
        for c in range(nRc):
            H = np.exp(gl[c]) * H + Sf[c]
        Hr = H.copy()
        Hf, Hb = [None] * nVc, [None] * nVc
        for v in range(nVc):
            Hf[v] = _r(H)
            H = np.exp(gl[nRc + v]) * H + Sf[nRc + v]
        H = Hr
        for v in range(nVc - 1, -1, -1):
            Hb[v] = _r(H)
            H = np.exp(gl[nRc + v]) * H + Sb[nRc + v]
        for v in range(nVc):
            a0, a1 = chunks[nRc + v]
            m = a1 - a0
            a = delta[a0:a1, h] * A[h]
            s = np.cumsum(a)
            sx = s - a
            G = Cm[a0:a1] @ Bm[a0:a1].T
            i = np.arange(m)[:, None]
            j = np.arange(m)[None, :]
            dec = np.where(j < i, np.exp(np.minimum(s[:, None] - s[None, :], 0)),
                           np.where(j > i, np.exp(np.minimum(sx[None, :] - sx[:, None], 0)), 0.0))
            M = _r(_r(G) * delta[a0:a1, h][None, :] * dec)
            y = M @ x[a0:a1, h] + np.exp(s)[:, None] * (Cm[a0:a1] @ Hf[v].T) + \
                np.exp(s[-1] - sx)[:, None] * (Cm[a0:a1] @ Hb[v].T)
            y += 2 * (np.diag(G) * delta[a0:a1, h] + D[h])[:, None] * x[a0:a1, h]
            out[v * Q:v * Q + m, h] = _r(y)
    return out


def elementwise_err(a, ref):
    """max_i |a_i - ref_i| / max(|ref_i|, rms(ref))."""
    a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    return float((np.abs(a - ref) / np.maximum(np.abs(ref), rms)).max())


def bf16_storage_forward_extras(X, w, cfg, layer):
    """bf16_storage_forward for the block with the Mamba2 extras: besides the block's own storage points,
    the convolved x | B | C rows, the gate z and the normalised rows are stored in bf16."""
    from oracle import mamba2_extras as MX
    order, shifted = layer % 4, layer % 2 == 1
    nP, N = cfg.nh * cfg.P, cfg.N
    outs = []
    for b in range(X.shape[0]):
        X3 = np.asarray(X[b], np.float64)
        T, H, W, d = X3.shape
        Xp = O.rms_permute(X3, order)
        Rv = _r(O.review_tokens(X3, cfg.R, order))
        S = np.concatenate([Rv, Xp], axis=0)
        x, Bm, Cm, delta = O.in_projection(S, w, cfg)
        xbc = _r(np.concatenate([x.reshape(-1, nP), Bm, Cm], axis=1))
        xbc = _r(MX.silu(MX.causal_conv(xbc, w["conv_w"], w["conv_b"])))
        x, Bm, Cm = xbc[:, :nP].reshape(-1, cfg.nh, cfg.P), xbc[:, nP:nP + N], xbc[:, nP + N:]
        A = -np.exp(np.asarray(w["A_log"], np.float64))
        y = _r(O.ssd_bidirectional(x, Bm, Cm, delta, A, w["D"], cfg.R).reshape(T * H * W, -1))
        z = _r(Xp @ np.asarray(w["W_z"], np.float64).T)
        yn = _r(MX.gated_rmsnorm(y, z, w["norm_w"]))
        ma = O.rms_unpermute(yn @ np.asarray(w["W_out"], np.float64).T, order, T, H, W)
        qkv = _r(X3.reshape(-1, d) @ np.asarray(w["W_qkv"], np.float64).T)
        Oa = _r(O.tesa_attention(qkv.reshape(T, H, W, -1), cfg.th, cfg.tp, (cfg.wt, cfg.wh, cfg.ww),
                                 (cfg.st, cfg.sh, cfg.sw), shifted))
        te = (Oa.reshape(-1, cfg.th * cfg.tp) @ np.asarray(w["W_o"], np.float64).T).reshape(T, H, W, d)
        outs.append(_r(ma + te))
    return np.stack(outs)
