"""Pins of the backward oracle (oracle/backward.py) to central finite differences of the forward oracle:
for a random output weighting G and a random direction V per input, <grad, V> must equal
(f(theta + eps V) - f(theta - eps V)) / (2 eps) with f = <forward(theta), G>, in fp64.  A dropped term, a
wrong sign or index, or a transposed operand anywhere in an adjoint moves that directional derivative by
far more than the central difference's O(eps^2) error.  CPU only."""
import numpy as np
import pytest

from mate_inputs import MateConfig, make_inputs
from oracle import backward as BW
from oracle import mate_oracle as O

EPS = 1e-5


def _fd(f, args, i, V):
    """Central difference of scalar f along direction V of argument i."""
    plus = list(args)
    minus = list(args)
    plus[i] = np.asarray(args[i], np.float64) + EPS * V
    minus[i] = np.asarray(args[i], np.float64) - EPS * V
    return (f(*plus) - f(*minus)) / (2 * EPS)


def _check(got, fd, what):
    assert abs(got - fd) <= 1e-6 * max(1.0, abs(fd)), f"{what}: adjoint {got!r} vs finite difference {fd!r}"


def _scan_case(seed, L=13, nh=2, P=3, N=4):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((L, nh, P)), rng.standard_normal((L, N)), rng.standard_normal((L, N)),
            O.softplus(rng.standard_normal((L, nh))), -np.exp(rng.uniform(-1, 0.5, nh)), rng.standard_normal(nh))


def test_recurrence_backward_matches_finite_differences():
    args = _scan_case(1)
    rng = np.random.default_rng(2)
    G = rng.standard_normal((13, 2, 3))
    grads = BW.ssd_recurrence_backward(*args, G)
    f = lambda *a: float(np.sum(O.ssd_recurrence(*a) * G))
    for i, name in enumerate(("x", "B", "C", "delta", "A", "D")):
        V = rng.standard_normal(np.shape(args[i]))
        _check(float(np.sum(grads[i] * V)), _fd(f, args, i, V), f"recurrence d{name}")


@pytest.mark.parametrize("R", [0, 4])
def test_bidirectional_backward_matches_finite_differences(R):
    args = _scan_case(3)
    rng = np.random.default_rng(4)
    G = rng.standard_normal((13 - R, 2, 3))
    grads = BW.ssd_bidirectional_backward(*args, R, G)
    f = lambda *a: float(np.sum(O.ssd_bidirectional(*a, R) * G))
    for i, name in enumerate(("x", "B", "C", "delta", "A", "D")):
        V = rng.standard_normal(np.shape(args[i]))
        _check(float(np.sum(grads[i] * V)), _fd(f, args, i, V), f"bidirectional R={R} d{name}")


def test_backward_of_the_decay_free_scan_is_a_reverse_cumulative_sum():
    """A = 0, D = 0, one head, P = N = 1, B = C = 1: y_t = sum_{s<=t} delta_s x_s, so dx_s = delta_s *
    sum_{t>=s} dy_t, a reverse cumulative sum written out directly."""
    rng = np.random.default_rng(5)
    L = 9
    x = rng.standard_normal((L, 1, 1))
    delta = rng.uniform(0.1, 1.0, (L, 1))
    dy = rng.standard_normal((L, 1, 1))
    dx = BW.ssd_recurrence_backward(x, np.ones((L, 1)), np.ones((L, 1)), delta, np.zeros(1), np.zeros(1), dy)[0]
    want = delta[:, 0] * np.cumsum(dy[::-1, 0, 0])[::-1]
    np.testing.assert_allclose(dx[:, 0, 0], want, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("shifted", [False, True])
def test_tesa_backward_matches_finite_differences(shifted):
    rng = np.random.default_rng(6)
    T, H, W, th, tp = 4, 4, 4, 2, 3
    win, sh = (2, 2, 2), (1, 1, 1)
    qkv = rng.standard_normal((T, H, W, 3 * th * tp))
    G = rng.standard_normal((T, H, W, th * tp))
    grad = BW.tesa_attention_backward(qkv, th, tp, win, sh, shifted, G)
    f = lambda a: float(np.sum(O.tesa_attention(a, th, tp, win, sh, shifted) * G))
    for trial in range(3):
        V = rng.standard_normal(qkv.shape)
        _check(float(np.sum(grad * V)), _fd(f, [qkv], 0, V), f"tesa shifted={shifted} trial {trial}")


def test_tesa_backward_of_a_single_key_is_the_output_gradient():
    """Window of one token: attention returns v, so dv = dO and dq = dk = 0."""
    rng = np.random.default_rng(7)
    qkv = rng.standard_normal((2, 2, 2, 3 * 2 * 3))
    dO = rng.standard_normal((2, 2, 2, 6))
    g = BW.tesa_attention_backward(qkv, 2, 3, (1, 1, 1), (0, 0, 0), False, dO)
    np.testing.assert_array_equal(g[..., :12], 0.0)
    np.testing.assert_allclose(g[..., 12:], dO, rtol=0, atol=0)


def _tiny_cfg(R=16):
    return MateConfig("t", 1, 2, 4, 4, 8, 2, 4, 3, 8, R, 2, 4, 2, 2, 2, 1, 1, 1, "f32", 0)


@pytest.mark.parametrize("layer", [0, 1, 2, 3])
def test_block_backward_matches_finite_differences(layer):
    cfg = _tiny_cfg()
    w = {k: np.asarray(v, np.float64) for k, v in make_inputs(cfg).items()}
    w["dt_bias"] = np.array([0.3, -0.2])
    rng = np.random.default_rng(10 + layer)
    G = rng.standard_normal(w["X"].shape)
    dX, grads = BW.mate_backward(w["X"], w, cfg, layer, G)
    f_of = lambda key: (lambda val: float(np.sum(O.mate_forward(
        val if key == "X" else w["X"], w if key == "X" else dict(w, **{key: val}), cfg, layer) * G)))
    for key in ("X", "W_in", "dt_bias", "A_log", "D", "W_out", "W_qkv", "W_o"):
        V = rng.standard_normal(np.shape(w[key]))
        got = float(np.sum((dX if key == "X" else grads[key]) * V))
        _check(got, _fd(f_of(key), [w[key]], 0, V), f"block layer {layer} d{key}")


def test_block_backward_without_review_tokens():
    cfg = _tiny_cfg(R=0)
    w = {k: np.asarray(v, np.float64) for k, v in make_inputs(cfg).items()}
    rng = np.random.default_rng(20)
    G = rng.standard_normal(w["X"].shape)
    dX, _ = BW.mate_backward(w["X"], w, cfg, 2, G)
    V = rng.standard_normal(w["X"].shape)
    f = lambda x: float(np.sum(O.mate_forward(x, w, cfg, 2) * G))
    _check(float(np.sum(dX * V)), _fd(f, [w["X"]], 0, V), "block R=0 dX")
