"""Backward pass of TEmporal Swin Attention (tesa_backward, through the C ABI) against the fp64 backward
oracle (oracle/backward.py, pinned by finite differences of the forward oracle), element by element.

Inputs: qkv and the output gradient dO ~ N(0, 1) rounded to bf16; the forward output O that the backward
reads comes from the library's own forward (tesa_forward) on the same qkv, as in training.  Criterion: the
intermediate entry points' element-wise bound, max(2e-2, 1.5 x the storage floor), the floor being the
oracle gradient rounded to bf16 (the entry point's only stored tensor); plus the relative bound."""
import numpy as np
import pytest

from helpers import assert_close_elementwise, oracle_cached, requires_gpu
from bf16_floor import elementwise_err, round_bf16
import mate_inputs as mi
from edge_configs import all_test_configs

pytestmark = [pytest.mark.gpu, requires_gpu]

torch = pytest.importorskip("torch")
from linear_complexity_video_mate_b200 import mate as M  # noqa: E402
from oracle import backward as BW  # noqa: E402

BW_SRC = ("oracle/backward.py",)
NAMES = ["bf16_small_8x16x16", "bf16_ragged_12x16x24", "bf16_b2_20x16x16_d512", "bf16_onechunk_4x8x8",
         "bf16_16x32x32"]


@pytest.mark.parametrize("shifted", [False, True])
@pytest.mark.parametrize("name", NAMES)
def test_tesa_backward(name, shifted):
    cfg = all_test_configs()[name]
    rng = np.random.default_rng(70 + len(name))
    a = cfg.th * cfg.tp
    qkv = mi.round_to_bf16(rng.standard_normal((cfg.B, cfg.T, cfg.H, cfg.W, 3 * a)))
    dO = mi.round_to_bf16(rng.standard_normal((cfg.B, cfg.T, cfg.H, cfg.W, a)))
    q_d = torch.as_tensor(qkv).to(device="cuda", dtype=torch.bfloat16)
    dO_d = torch.as_tensor(dO).to(device="cuda", dtype=torch.bfloat16)
    O_d = M.tesa_forward(q_d, shifted, cfg)
    got = M.tesa_backward(q_d, O_d, dO_d, shifted, cfg).float().cpu().numpy()
    ref = oracle_cached(f"tesa-bwd-{name}-{shifted}", lambda: np.stack([
        BW.tesa_attention_backward(qkv[b], cfg.th, cfg.tp, (cfg.wt, cfg.wh, cfg.ww), (cfg.st, cfg.sh, cfg.sw),
                                   shifted, dO[b]) for b in range(cfg.B)]), BW_SRC)
    for part, sl in (("dq", slice(0, a)), ("dk", slice(a, 2 * a)), ("dv", slice(2 * a, 3 * a))):
        g, r = got[..., sl], ref[..., sl]
        assert_close_elementwise(g, r, "bf16", f"tesa backward {name} shifted={shifted} {part}",
                                 elementwise_err(round_bf16(r), r))
    assert M.device_status() == 0
