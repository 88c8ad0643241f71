"""Parity of the block with the rest of the Mamba2 block around the scan (causal depthwise convolution +
SiLU on x | B | C, SiLU(z) gate, gated RMSNorm) against oracle.mamba2_extras, element by element on seeded
inputs.  The pages name the MA branch's core a bidirectional Mamba2 block without listing its parts."""
import math

import numpy as np
import pytest

from helpers import assert_close, oracle_cached, requires_gpu
from bf16_floor import bf16_storage_forward_extras, rms_normalised_max_err
import mate_inputs as mi
from edge_configs import all_test_configs
from oracle import mamba2_extras as MX

pytestmark = [pytest.mark.gpu, requires_gpu]

torch = pytest.importorskip("torch")
from linear_complexity_video_mate_b200 import mate as M  # noqa: E402
from test_gpu_parity import dev, host, tdt  # noqa: E402

MX_SRC = ("oracle/mamba2_extras.py",)
NAMES = ["tiny_f32_4x8x8", "f32_b2_4x8x12", "bf16_small_8x16x16", "bf16_ragged_12x16x24", "bf16_onechunk_4x8x8",
         "bf16_noreview_b2_8x16x16", "bf16_b2_20x16x16_d512"]


def extras_weights(cfg, seed):
    """Gate projection N(0, 1/d); convolution taps and bias U(-1/2, 1/2) (the default initialisation of a
    width-4 depthwise convolution); norm weight 1 + N(0, 0.1^2)."""
    rng = np.random.default_rng(seed)
    nP, Cx = cfg.nh * cfg.P, cfg.nh * cfg.P + 2 * cfg.N
    W_z = rng.standard_normal((nP, cfg.d)) / math.sqrt(cfg.d)
    if cfg.dtype == "bf16":
        W_z = mi.round_to_bf16(W_z)
    return dict(W_z=np.asarray(W_z, np.float32),
                conv_w=rng.uniform(-0.5, 0.5, (Cx, MX.CONV_K)).astype(np.float32),
                conv_b=rng.uniform(-0.5, 0.5, Cx).astype(np.float32),
                norm_w=(1.0 + 0.1 * rng.standard_normal(nP)).astype(np.float32))


def block_reference(name, layer, variant="default"):
    """(weights, sampled output rows, oracle output on them, bf16 storage floor on the same rows)."""
    cfg = all_test_configs()[name]
    w = dict(mi.make_inputs(cfg))
    w.update(extras_weights(cfg, 41))
    if variant == "maonly":
        w["W_o"] = np.zeros_like(w["W_o"])
    rows = np.unique(np.append(np.arange(0, cfg.B * cfg.n, 16), cfg.B * cfg.n - 1))
    key = f"mx-mate-{name}-{layer}-{variant}-every16"
    ref = oracle_cached(key, lambda: MX.mate_forward_extras(w["X"], w, cfg, layer).reshape(
        cfg.B * cfg.n, cfg.d)[rows], MX_SRC)
    floor = 0.0
    if cfg.dtype == "bf16":
        floor = float(oracle_cached(f"mx-floor-{key}", lambda: np.array([rms_normalised_max_err(
            bf16_storage_forward_extras(w["X"], w, cfg, layer).reshape(cfg.B * cfg.n, cfg.d)[rows], ref)]),
            MX_SRC)[0])
    return w, rows, ref, floor


CASES = [(n, l, "default") for n in NAMES for l in range(4)] + \
        [(n, l, "maonly") for n in ("bf16_small_8x16x16", "bf16_ragged_12x16x24") for l in (0, 3)]


@pytest.mark.parametrize("name,layer,variant", CASES)
def test_mate_forward_extras(name, layer, variant):
    cfg = all_test_configs()[name]
    w, rows, ref, floor = block_reference(name, layer, variant)
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    assert blk.extras
    out = host(blk.forward(dev(w["X"], tdt(cfg)), layer)).reshape(cfg.B * cfg.n, cfg.d)[rows]
    assert_close(out, ref, cfg.dtype, f"extras mate {name} layer {layer} {variant}", floor)


def test_extras_host_path_matches_device_path():
    cfg = all_test_configs()["bf16_b2_20x16x16_d512"]
    w = dict(mi.make_inputs(cfg))
    w.update(extras_weights(cfg, 42))
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    Xd = dev(w["X"], torch.bfloat16)
    ref = blk.forward(Xd, 2)
    xh = Xd.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    blk.forward_host(xh, 2, oh)
    torch.cuda.synchronize()
    assert torch.equal(oh, ref.cpu())


def test_extras_change_the_output_and_leave_the_device_status_clean():
    """The extras are not a no-op: the same block without them gives a different output."""
    cfg = all_test_configs()["bf16_small_8x16x16"]
    w = dict(mi.make_inputs(cfg))
    Xd = dev(w["X"], torch.bfloat16)
    plain = M.MateBlock(cfg, M.weights_to_device(w, cfg)).forward(Xd, 1).float()
    w.update(extras_weights(cfg, 43))
    full = M.MateBlock(cfg, M.weights_to_device(w, cfg)).forward(Xd, 1).float()
    assert (full - plain).abs().max().item() > 1e-2 * plain.abs().max().item()
    assert M.device_status() == 0


def test_extras_weights_must_come_together():
    cfg = all_test_configs()["tiny_f32_4x8x8"]
    w = dict(mi.make_inputs(cfg))
    w["W_z"] = extras_weights(cfg, 44)["W_z"]
    with pytest.raises(ValueError):
        M.MateBlock(cfg, M.weights_to_device(w, cfg))
