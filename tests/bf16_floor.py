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
