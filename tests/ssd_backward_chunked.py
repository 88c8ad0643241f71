"""Chunked formulation of the selective scan's backward pass: the decomposition a tensor-core backward
kernel computes, in exact fp64 arithmetic, checked against the sequential adjoint of oracle/backward.py.

Test-side emulation (like the chunked forward emulation in bf16_floor.py), not part of the oracle.

For one head and one direction, with a_t = delta_t A, s the within-chunk inclusive cumulative sum of a,
H_c the state entering chunk c and E_c the adjoint arriving at chunk c's last row from the chunks after it:
  forward carry   H_{c+1} = exp(s_last) H_c + sum_j exp(s_last - s_j) delta_j x_j B_j^T
  adjoint carry   E_{c-1} = exp(s_last) E_c + sum_k exp(s_k) dy_k C_k^T          (right to left)
  inside a chunk (i, j, k rows of it):
    dx_i  = delta_i [ sum_{k>=i} exp(s_k - s_i) (B_i . C_k) dy_k + exp(s_last - s_i) E_c B_i ] + D dy_i
    dB_i  = delta_i [ sum_{k>=i} exp(s_k - s_i) (x_i . dy_k) C_k + exp(s_last - s_i) E_c^T x_i ]
    dC_k  = sum_{j<=k} exp(s_k - s_j) delta_j (dy_k . x_j) B_j + exp(s_k) H_c^T dy_k
  so dx is the reverse-direction scan with B and C swapped and delta applied to the output, and dB, dC
  are the same Q x Q matrix shapes as the forward's M.  The log-decay gradient da_m (a_m = delta_m A) is
  the sum of W_kj = (dy_k . x_j)(C_k . B_j) delta_j exp(s_k - s_j) over the pairs j < m <= k, which
  splits into four chunk-local pieces: pairs inside the chunk (a 2D straddle sum of the Q x Q matrix W),
  H_c against rows k >= m (a reverse cumulative sum), rows j < m against E_c (a prefix sum), and
  exp(s_last) <H_c, E_c> for every row.  Then ddelta_m = x_m . (G_m B_m) + A da_m and dA = sum delta_m da_m.
"""
from __future__ import annotations

import numpy as np


def _chunks(L: int, Q: int):
    return [(c0, min(c0 + Q, L)) for c0 in range(0, L, Q)]


def ssd_backward_chunked(x, Bm, Cm, delta, A, D, dy, Q: int, chunks=None):
    """Gradients of the one-direction recurrence (same outputs as oracle.backward.ssd_recurrence_backward)
    computed chunk by chunk.  x [L, nh, P], Bm / Cm [L, N], delta [L, nh], A / D [nh], dy [L, nh, P].
    `chunks` (a list of [c0, c1) covering 0..L in order) overrides the uniform cut into Q rows."""
    x, Bm, Cm, delta, A, D, dy = (np.asarray(v, np.float64) for v in (x, Bm, Cm, delta, A, D, dy))
    L, nh, P = x.shape
    N = Bm.shape[1]
    chunks = _chunks(L, Q) if chunks is None else list(chunks)
    dx, dB, dC = np.zeros_like(x), np.zeros_like(Bm), np.zeros_like(Cm)
    ddelta, dA, dD = np.zeros_like(delta), np.zeros(nh), np.zeros(nh)
    for h in range(nh):
        a = delta[:, h] * A[h]
        s = [np.cumsum(a[c0:c1]) for c0, c1 in chunks]
        # forward carry: state entering each chunk
        Hin = [np.zeros((P, N))]
        for c, (c0, c1) in enumerate(chunks[:-1]):
            w = np.exp(s[c][-1] - s[c]) * delta[c0:c1, h]
            Hin.append(np.exp(s[c][-1]) * Hin[c] + (w[:, None] * x[c0:c1, h]).T @ Bm[c0:c1])
        # adjoint carry, right to left: E[c] arrives at chunk c's last row
        E = [None] * len(chunks)
        E[-1] = np.zeros((P, N))
        for c in range(len(chunks) - 1, 0, -1):
            c0, c1 = chunks[c]
            E[c - 1] = np.exp(s[c][-1]) * E[c] + (np.exp(s[c])[:, None] * dy[c0:c1, h]).T @ Cm[c0:c1]
        for c, (c0, c1) in enumerate(chunks):
            sc, sl = s[c], s[c][-1]
            xs, dys, Bs, Cs, dl = x[c0:c1, h], dy[c0:c1, h], Bm[c0:c1], Cm[c0:c1], delta[c0:c1, h]
            m = c1 - c0
            i = np.arange(m)[:, None]
            k = np.arange(m)[None, :]
            up = np.where(k >= i, np.exp(np.minimum(sc[None, :] - sc[:, None], 0.0)), 0.0)   # [i, k], k >= i
            lo = up.T                                                                     # [k, j], j <= k
            # dx: reverse scan with B and C swapped
            gB = (up * (Bs @ Cs.T)) @ dys + np.exp(sl - sc)[:, None] * (Bs @ E[c].T)      # (G_i B_i) [m, P]
            dx[c0:c1, h] = dl[:, None] * gB + D[h] * dys
            # dB: the same matrix shape with x . dy
            dB[c0:c1] += dl[:, None] * ((up * (xs @ dys.T)) @ Cs + np.exp(sl - sc)[:, None] * (xs @ E[c]))
            # dC: forward-shaped matrix with dy . x
            dC[c0:c1] += (lo * (dys @ xs.T) * dl[None, :]) @ Bs + np.exp(sc)[:, None] * (dys @ Hin[c])
            dD[h] += np.sum(xs * dys)
            # da_m: straddle sums of W_kj over j < m <= k
            W = lo * (dys @ xs.T) * (Cs @ Bs.T) * dl[None, :]          # [k, j], j <= k (diagonal included)
            np.fill_diagonal(W, 0.0)                                  # pairs need j < m <= k, so j < k
            inside = np.array([W[mm:, :mm].sum() for mm in range(m)])
            q = np.exp(sc) * np.einsum("kp,pn,kn->k", dys, Hin[c], Cs)
            from_h = np.cumsum(q[::-1])[::-1]                          # sum over k >= m
            pj = np.exp(sl - sc) * dl * np.einsum("jp,pn,jn->j", xs, E[c], Bs)
            to_e = np.concatenate([[0.0], np.cumsum(pj)[:-1]])         # sum over j < m
            both = np.exp(sl) * np.sum(Hin[c] * E[c])
            da = inside + from_h + to_e + both
            ddelta[c0:c1, h] = np.sum(xs * gB, axis=1) + A[h] * da
            dA[h] += np.sum(dl * da)
    return dx, dB, dC, ddelta, dA, dD


def kernel_chunks(R: int, n: int, Q: int, backward: bool):
    """The chunk boundaries the tensor-core scan uses over [review rows; video rows]: ceil(R/Q) review
    chunks, then the video rows cut at multiples of Q of the scan position.  The backward traversal runs
    over [review rows; video rows reversed] and visits the same video chunks in reverse order, so in its
    own coordinates a partial last video chunk comes first."""
    out = [(c0, min(c0 + Q, R)) for c0 in range(0, R, Q)]
    video = [(v0, min(v0 + Q, n)) for v0 in range(0, n, Q)]
    if backward:
        video = [(n - v1, n - v0) for v0, v1 in reversed(video)]
    return out + [(R + a, R + b) for a, b in video]


def ssd_bidirectional_backward_chunked(x, Bm, Cm, delta, A, D, R: int, dy, Q: int):
    """Gradients of the bidirectional scan with a prefix (the same outputs as
    oracle.backward.ssd_bidirectional_backward), each direction computed chunk by chunk on the chunks the
    forward kernels use: the forward direction over [prefix; video], the backward direction over [prefix;
    video reversed] with its per-row gradients mapped back through the flip."""
    x = np.asarray(x, np.float64)
    L, nh, P = x.shape
    n = L - R
    dy = np.asarray(dy, np.float64)
    dyf = np.zeros((L, nh, P))
    dyf[R:] = dy
    gf = ssd_backward_chunked(x, Bm, Cm, delta, A, D, dyf, Q, kernel_chunks(R, n, Q, False))
    flip = np.concatenate([np.arange(R), np.arange(L - 1, R - 1, -1)])
    dyb = np.zeros((L, nh, P))
    dyb[R:] = dy[::-1]
    Bm, Cm, delta = (np.asarray(v, np.float64) for v in (Bm, Cm, delta))
    gb = ssd_backward_chunked(x[flip], Bm[flip], Cm[flip], delta[flip], A, D, dyb, Q, kernel_chunks(R, n, Q, True))
    out = []
    for f, b in zip(gf[:4], gb[:4]):
        g = f.copy()
        g[flip] += b
        out.append(g)
    return out[0], out[1], out[2], out[3], gf[4] + gb[4], gf[5] + gb[5]

