"""Parity of the scan and the whole block with separate backward-direction scan parameters (dt_bias_b,
A_log_b, D_b) against oracle.per_direction, element by element on seeded inputs.  The pages leave open
whether the two directions of the bidirectional Mamba2 block share these parameters; the library runs
either reading, and with the backward parameters equal to the forward ones the per-direction path must
give what the shared path gives."""
import numpy as np
import pytest

from helpers import assert_close, assert_close_elementwise, oracle_cached, requires_gpu
from bf16_floor import bf16_storage_forward, rms_normalised_max_err
import mate_inputs as mi
from edge_configs import all_test_configs
from oracle import mate_oracle as O
from oracle import per_direction as PD

pytestmark = [pytest.mark.gpu, requires_gpu]

torch = pytest.importorskip("torch")
from linear_complexity_video_mate_b200 import mate as M  # noqa: E402
from test_gpu_parity import _ssd_floor, _ssd_inputs, dev, host, tdt  # noqa: E402

PD_SRC = ("oracle/per_direction.py",)
NAMES = ["tiny_f32_4x8x8", "f32_b2_4x8x12", "bf16_small_8x16x16", "bf16_ragged_12x16x24", "bf16_onechunk_4x8x8",
         "bf16_noreview_b2_8x16x16"]


def backward_params(nh, seed, dt_bias, a_log_range):
    """Backward-scan parameters drawn beside the forward ones: step-size bias within +-1 of the forward
    bias, A_log over the same range, D ~ N(0, 1)."""
    rng = np.random.default_rng(seed)
    dt_bias_b = (np.asarray(dt_bias, np.float64) + rng.uniform(-1.0, 1.0, nh)).astype(np.float32)
    A_log_b = rng.uniform(a_log_range[0], a_log_range[1], nh).astype(np.float32)
    D_b = rng.standard_normal(nh).astype(np.float32)
    return dt_bias_b, A_log_b, D_b


def _pd_oracle(cfg, x, Bm, Cm, dt, dt_bias, A_log, D, dt_bias_b, A_log_b, D_b):
    out = []
    for b in range(cfg.B):
        xs = x[b].reshape(-1, cfg.nh, cfg.P)
        dt64 = dt[b].astype(np.float64)
        out.append(PD.ssd_bidirectional_per_direction(
            xs, Bm[b], Cm[b], O.softplus(dt64 + dt_bias.astype(np.float64)), -np.exp(A_log.astype(np.float64)),
            D.astype(np.float64), O.softplus(dt64 + dt_bias_b.astype(np.float64)),
            -np.exp(A_log_b.astype(np.float64)), D_b.astype(np.float64), cfg.R))
    return np.stack(out)


def _scan_args(cfg, long_memory):
    args = _ssd_inputs(cfg, long_memory, 27)
    rng_range = (-3.0, -1.0) if long_memory else (0.0, 1.0)
    bwd = backward_params(cfg.nh, 28, args[4], rng_range)
    return args, bwd


def _pd_scan(cfg, args, bwd):
    x, Bm, Cm, dt, dt_bias, A_log, D = args
    td = tdt(cfg)
    f32 = torch.float32
    return M.ssd_scan_bidir_pd(dev(x, td), dev(Bm, td), dev(Cm, td), dev(dt, f32), dev(dt_bias, f32), dev(A_log, f32),
                               dev(D, f32), *(dev(a, f32) for a in bwd), cfg.R, cfg)


def video_rows(cfg, stride=16):
    """Every stride-th video row plus the last one: the rows whose oracle values are kept on disk (the GPU
    computes all of them; the stored references stay small)."""
    return np.unique(np.append(np.arange(0, cfg.n, stride), cfg.n - 1))


def scan_reference(name, long_memory):
    """(inputs, backward parameters, sampled rows, oracle y on those rows, bf16 storage floor) of the
    per-direction scan case.  The floor is that of the stored bf16 output on the same rows."""
    cfg = all_test_configs()[name]
    args, bwd = _scan_args(cfg, long_memory)
    rows = video_rows(cfg)
    key = f"pd-ssd-{name}-{long_memory}-every16"
    ref = oracle_cached(key, lambda: _pd_oracle(cfg, *args, *bwd)[:, rows], PD_SRC)
    return args, bwd, rows, ref, _ssd_floor(cfg, ref)


@pytest.mark.parametrize("long_memory", [False, True])
@pytest.mark.parametrize("name", NAMES)
def test_ssd_scan_per_direction(name, long_memory):
    cfg = all_test_configs()[name]
    args, bwd, rows, ref, floor = scan_reference(name, long_memory)
    got = host(_pd_scan(cfg, args, bwd)).reshape(cfg.B, cfg.n, cfg.nh, cfg.P)[:, rows]
    assert_close_elementwise(got, ref, cfg.dtype, f"pd ssd {name} long={long_memory}", floor)


@pytest.mark.parametrize("name", ["tiny_f32_4x8x8", "bf16_small_8x16x16", "bf16_noreview_b2_8x16x16"])
def test_ssd_scan_per_direction_with_shared_values_matches_shared_path(name):
    """Backward parameters equal to the forward ones: the per-direction kernels take the same decisions
    on the same values, so the result matches the shared-parameter entry point to within one rounding of
    the stored output."""
    cfg = all_test_configs()[name]
    args, _ = _scan_args(cfg, False)
    x, Bm, Cm, dt, dt_bias, A_log, D = args
    td = tdt(cfg)
    f32 = torch.float32
    shared = host(M.ssd_scan_bidir(dev(x, td), dev(Bm, td), dev(Cm, td), dev(dt, f32), dev(dt_bias, f32),
                                   dev(A_log, f32), dev(D, f32), cfg.R, cfg))
    pd = host(_pd_scan(cfg, args, (dt_bias, A_log, D)))
    ulp = 2.0 ** -8 if cfg.dtype == "bf16" else 1e-6
    rms = np.sqrt(np.mean(shared.astype(np.float64) ** 2))
    assert (np.abs(pd - shared) <= ulp * np.maximum(np.abs(shared), rms)).all(), name


BLOCK_NAMES = ["tiny_f32_4x8x8", "bf16_small_8x16x16", "bf16_ragged_12x16x24", "bf16_noreview_b2_8x16x16"]


def block_reference(name, layer):
    """(weights with backward parameters, sampled output rows, oracle output on them, bf16 storage floor)
    of the block case; the floor is the larger of the shared-parameter floors with either direction's
    parameters, on the same rows."""
    cfg = all_test_configs()[name]
    w = dict(mi.make_inputs(cfg))
    w["dt_bias_b"], w["A_log_b"], w["D_b"] = backward_params(cfg.nh, 29, w["dt_bias"], (0.0, 1.0))
    rows = np.unique(np.append(np.arange(0, cfg.B * cfg.n, 16), cfg.B * cfg.n - 1))
    key = f"pd-mate-{name}-{layer}-every16"
    ref = oracle_cached(key, lambda: PD.mate_forward_per_direction(w["X"], w, cfg, layer).reshape(
        cfg.B * cfg.n, cfg.d)[rows], PD_SRC)
    floor = 0.0
    if cfg.dtype == "bf16":
        for tag, wb in (("f", w), ("b", dict(w, dt_bias=w["dt_bias_b"], A_log=w["A_log_b"], D=w["D_b"]))):
            def fl(wb=wb):
                r = O.mate_forward(wb["X"], wb, cfg, layer).reshape(cfg.B * cfg.n, cfg.d)[rows]
                return np.array([rms_normalised_max_err(
                    bf16_storage_forward(wb["X"], wb, cfg, layer).reshape(cfg.B * cfg.n, cfg.d)[rows], r)])
            floor = max(floor, float(oracle_cached(f"pd-floor-{key}-{tag}", fl, PD_SRC)[0]))
    return w, rows, ref, floor


@pytest.mark.parametrize("layer", [0, 1, 2, 3])
@pytest.mark.parametrize("name", BLOCK_NAMES)
def test_mate_forward_per_direction(name, layer):
    cfg = all_test_configs()[name]
    w, rows, ref, floor = block_reference(name, layer)
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    out = host(blk.forward(dev(w["X"], tdt(cfg)), layer)).reshape(cfg.B * cfg.n, cfg.d)[rows]
    assert_close(out, ref, cfg.dtype, f"pd mate {name} layer {layer}", floor)


def test_mate_block_rejects_partial_backward_parameters():
    cfg = all_test_configs()["tiny_f32_4x8x8"]
    w = dict(mi.make_inputs(cfg))
    w["A_log_b"] = w["A_log"]
    with pytest.raises(ValueError):
        M.MateBlock(cfg, M.weights_to_device(w, cfg))
