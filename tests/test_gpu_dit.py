"""The DiT block around MATE (mate_dit_block_forward, through the C ABI) against the fp64 oracle of
oracle/dit_block.py: adaLN-Zero modulation, the mixer behind a gated residual, the gated GELU MLP.  fp32
blocks at 1e-4 relative; bf16 blocks at the block's bf16 criterion with the DiT block's own storage floor
(tests/bf16_floor.py, bf16_storage_dit)."""
import math

import numpy as np
import pytest

from helpers import assert_close, oracle_cached, requires_gpu
from bf16_floor import bf16_storage_dit, rms_normalised_max_err
import mate_inputs as mi
from edge_configs import all_test_configs

pytestmark = [pytest.mark.gpu, requires_gpu]

torch = pytest.importorskip("torch")
from linear_complexity_video_mate_b200 import mate as M  # noqa: E402
from oracle import dit_block as DB  # noqa: E402

DC = 256                     # conditioning width (timestep + pooled text embedding)
DIT_SRC = ("oracle/dit_block.py",)


def dit_inputs(cfg, seed):
    """The block's inputs and MATE weights (mate_inputs) plus DiT weights: W_ada N(0, 1/dc), b_ada
    N(0, 0.1^2) (non-zero, so that every modulation path is exercised; adaLN-Zero starts training from
    zero), W1 N(0, 1/d), W2 N(0, 1/(4d)), biases N(0, 0.1^2), c N(0, 1); matrices rounded to bf16 for bf16
    blocks."""
    w = dict(mi.make_inputs(cfg))
    rng = np.random.default_rng(seed)
    d = cfg.d
    cast = (lambda a: mi.round_to_bf16(a)) if cfg.dtype == "bf16" else (lambda a: np.asarray(a, np.float32))
    w.update(W_ada=cast(rng.standard_normal((6 * d, DC)) / math.sqrt(DC)),
             b_ada=(0.1 * rng.standard_normal(6 * d)).astype(np.float32),
             W1=cast(rng.standard_normal((4 * d, d)) / math.sqrt(d)),
             b1=(0.1 * rng.standard_normal(4 * d)).astype(np.float32),
             W2=cast(rng.standard_normal((d, 4 * d)) / math.sqrt(4 * d)),
             b2=(0.1 * rng.standard_normal(d)).astype(np.float32))
    c = rng.standard_normal((cfg.B, DC)).astype(np.float32)
    return w, c


CASES = [("tiny_f32_4x8x8", l) for l in range(4)] + [("f32_b2_4x8x12", 1)] + \
        [("bf16_small_8x16x16", l) for l in range(4)] + [("bf16_b2_20x16x16_d512", 2), ("bf16_16x32x32", 1)]


@pytest.mark.parametrize("name,layer", CASES)
def test_dit_block_forward(name, layer):
    cfg = all_test_configs()[name]
    w, c = dit_inputs(cfg, 50 + layer)
    tdt = M.torch_dtype(cfg)
    blk = M.DitBlock(cfg, M.weights_to_device(w, cfg), M.dit_weights_to_device(w, cfg), DC)
    X = torch.as_tensor(w["X"]).to(device="cuda", dtype=tdt)
    out = blk.forward(X, torch.as_tensor(c).cuda(), layer).float().cpu().numpy()
    key = f"dit-{name}-{layer}"
    ref = oracle_cached(key, lambda: DB.dit_block(w["X"], c, w, cfg, layer), DIT_SRC)
    floor = 0.0
    if cfg.dtype == "bf16":
        floor = float(oracle_cached(f"floor-{key}", lambda: np.array([rms_normalised_max_err(
            bf16_storage_dit(w["X"], c, w, cfg, layer), ref)]), DIT_SRC)[0])
    assert_close(out, ref, cfg.dtype, f"dit {name} layer {layer}", floor)
    assert M.device_status() == 0


def test_dit_block_with_zero_modulation_passes_x_through():
    """adaLN-Zero at initialisation: zero modulation weights and biases make both gates zero, so the block
    returns X exactly (the gated residual epilogues add 0 x the branch to the stored residual)."""
    cfg = all_test_configs()["bf16_small_8x16x16"]
    w, c = dit_inputs(cfg, 60)
    w["W_ada"] = np.zeros_like(w["W_ada"])
    w["b_ada"] = np.zeros_like(w["b_ada"])
    blk = M.DitBlock(cfg, M.weights_to_device(w, cfg), M.dit_weights_to_device(w, cfg), DC)
    X = torch.as_tensor(w["X"]).to(device="cuda", dtype=torch.bfloat16)
    out = blk.forward(X, torch.as_tensor(c).cuda(), 1)
    assert torch.equal(out, X)
