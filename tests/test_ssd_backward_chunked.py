"""The chunked backward formulation (tests/ssd_backward_chunked.py) equals the sequential adjoint of the
backward oracle, for chunk lengths that divide the sequence, leave a ragged tail, cover it in one chunk
or are one row long.  CPU only."""
import numpy as np
import pytest

from oracle import backward as BW
from oracle import mate_oracle as O
from ssd_backward_chunked import ssd_backward_chunked


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
