"""The chunked backward formulation (tests/ssd_backward_chunked.py) equals the sequential adjoint of the
backward oracle, for chunk lengths that divide the sequence, leave a ragged tail, cover it in one chunk
or are one row long.  CPU only."""
import numpy as np
import pytest

from oracle import backward as BW
from oracle import mate_oracle as O
from ssd_backward_chunked import kernel_chunks, ssd_backward_chunked, ssd_bidirectional_backward_chunked


@pytest.mark.parametrize("Q", [1, 4, 7, 16, 64])
@pytest.mark.parametrize("decay", ["moderate", "fast"])
def test_chunked_backward_equals_sequential(Q, decay):
    rng = np.random.default_rng(Q)
    L, nh, P, N = 29, 2, 3, 4
    x = rng.standard_normal((L, nh, P))
    Bm, Cm = rng.standard_normal((L, N)), rng.standard_normal((L, N))
    delta = O.softplus(rng.standard_normal((L, nh)))
    A = -np.exp(rng.uniform(-1.0, 0.5, nh)) * (1.0 if decay == "moderate" else 20.0)
    D = rng.standard_normal(nh)
    dy = rng.standard_normal((L, nh, P))
    want = BW.ssd_recurrence_backward(x, Bm, Cm, delta, A, D, dy)
    got = ssd_backward_chunked(x, Bm, Cm, delta, A, D, dy, Q)
    for name, g, w in zip(("dx", "dB", "dC", "ddelta", "dA", "dD"), got, want):
        np.testing.assert_allclose(g, w, rtol=1e-11, atol=1e-11, err_msg=f"{name} Q={Q} {decay}")


@pytest.mark.parametrize("R,n,Q", [(0, 29, 8), (8, 29, 8), (12, 40, 8), (4, 7, 16), (16, 32, 16)])
def test_bidirectional_chunked_backward_on_kernel_chunks(R, n, Q):
    """Both directions on the forward kernels' own chunks (review chunks first; the backward direction's
    video chunks reversed, a partial one first), against the bidirectional adjoint of the backward oracle."""
    rng = np.random.default_rng(R + n + Q)
    L, nh, P, N = R + n, 2, 3, 4
    x = rng.standard_normal((L, nh, P))
    Bm, Cm = rng.standard_normal((L, N)), rng.standard_normal((L, N))
    delta = O.softplus(rng.standard_normal((L, nh)))
    A = -np.exp(rng.uniform(-1.0, 0.5, nh))
    D = rng.standard_normal(nh)
    dy = rng.standard_normal((n, nh, P))
    want = BW.ssd_bidirectional_backward(x, Bm, Cm, delta, A, D, R, dy)
    got = ssd_bidirectional_backward_chunked(x, Bm, Cm, delta, A, D, R, dy, Q)
    for name, g, w in zip(("dx", "dB", "dC", "ddelta", "dA", "dD"), got, want):
        np.testing.assert_allclose(g, w, rtol=1e-11, atol=1e-11, err_msg=f"{name} R={R} n={n} Q={Q}")


def test_kernel_chunks_cover_the_sequence_in_order():
    for R, n, Q in [(0, 29, 8), (12, 40, 8), (4, 7, 16)]:
        for bwd in (False, True):
            ch = kernel_chunks(R, n, Q, bwd)
            assert ch[0][0] == 0 and ch[-1][1] == R + n
            assert all(a[1] == b[0] for a, b in zip(ch, ch[1:])) and all(c1 > c0 for c0, c1 in ch)
    # the backward direction's first video chunk is the partial last one, reversed
    assert kernel_chunks(0, 29, 8, True)[0] == (0, 5)

