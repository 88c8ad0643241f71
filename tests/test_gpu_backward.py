"""The backward pass of the bidirectional scan (ssd_scan_bidir_backward, fp32 blocks) against the
backward oracle, element by element on seeded inputs, through the C ABI."""
import numpy as np
import pytest

from helpers import assert_close_elementwise, requires_gpu
from edge_configs import all_test_configs
from oracle import backward as BW
from oracle import mate_oracle as O

pytestmark = [pytest.mark.gpu, requires_gpu]

torch = pytest.importorskip("torch")
from linear_complexity_video_mate_b200 import mate as M  # noqa: E402
from test_gpu_parity import _ssd_inputs, dev, host  # noqa: E402


def _oracle(cfg, x, Bm, Cm, dt, dt_bias, A_log, D, dy):
    A = -np.exp(A_log.astype(np.float64))
    out = {k: [] for k in ("dx", "dB", "dC", "ddt")}
    dA_log, dD, ddt_bias = np.zeros(cfg.nh), np.zeros(cfg.nh), np.zeros(cfg.nh)
    for b in range(cfg.B):
        v = dt[b].astype(np.float64) + dt_bias.astype(np.float64)
        delta = O.softplus(v)
        gx, gB, gC, gd, gA, gD = BW.ssd_bidirectional_backward(
            x[b].reshape(-1, cfg.nh, cfg.P), Bm[b], Cm[b], delta, A, D.astype(np.float64), cfg.R,
            dy[b].reshape(cfg.n, cfg.nh, cfg.P))
        ddt = gd / (1.0 + np.exp(-v))
        out["dx"].append(gx.reshape(-1, cfg.nh * cfg.P))
        out["dB"].append(gB)
        out["dC"].append(gC)
        out["ddt"].append(ddt)
        dA_log += gA * A
        dD += gD
        ddt_bias += ddt.sum(axis=0)
    res = {k: np.stack(v) for k, v in out.items()}
    res.update(dA_log=dA_log, dD=dD, ddt_bias=ddt_bias)
    return res


@pytest.mark.parametrize("long_memory", [False, True])
@pytest.mark.parametrize("name", ["tiny_f32_4x8x8", "f32_b2_4x8x12"])
def test_ssd_scan_backward(name, long_memory):
    cfg = all_test_configs()[name]
    x, Bm, Cm, dt, dt_bias, A_log, D = _ssd_inputs(cfg, long_memory, 51)
    dy = np.random.default_rng(52).standard_normal((cfg.B, cfg.n, cfg.nh * cfg.P)).astype(np.float32)
    f32 = torch.float32
    g = M.ssd_scan_bidir_backward(dev(x, f32), dev(Bm, f32), dev(Cm, f32), dev(dt, f32), dev(dt_bias, f32),
                                  dev(A_log, f32), dev(D, f32), dev(dy, f32), cfg.R, cfg)
    ref = _oracle(cfg, x, Bm, Cm, dt, dt_bias, A_log, D, dy)
    for k in ("dx", "dB", "dC", "ddt"):
        assert_close_elementwise(host(g[k]), ref[k], "f32", f"backward {name} {k} long={long_memory}")
    for k in ("dA_log", "dD", "ddt_bias"):
        got, want = host(g[k]), ref[k]
        assert np.abs(got - want).max() <= 1e-4 * max(1.0, np.abs(want).max()), (k, got, want)
    assert M.device_status() == 0
