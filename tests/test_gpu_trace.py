"""The library's kernel-timing trace: one record per launch of a block forward, in launch order, with
positive device times."""
import pytest

from helpers import requires_gpu
import mate_inputs as mi

pytestmark = [pytest.mark.gpu, requires_gpu]

torch = pytest.importorskip("torch")
from linear_complexity_video_mate_b200 import mate as M  # noqa: E402


def test_trace_records_every_launch_of_a_forward():
    cfg = mi.TEST_CONFIGS["bf16_small_8x16x16"]
    w = mi.make_inputs(cfg)
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    X = torch.as_tensor(w["X"]).to(device="cuda", dtype=torch.bfloat16)
    out = torch.empty_like(X)
    blk.forward(X, 1, out)
    torch.cuda.synchronize()
    trace = M.KernelTrace(64).start()
    blk.forward(X, 1, out)
    trace.stop()
    recs = trace.read()
    assert len(recs) == M.MateBlock.last_launch_count()
    names = [n for n, _ in recs]
    for k in ("in_projection", "in_projection_review", "ssd_gram", "ssd_state", "ssd_carry", "ssd_output", "tesa",
              "out_projection"):
        assert names.count(k) == 1, names
    assert names.index("in_projection") < names.index("ssd_output") < names.index("out_projection")
    assert all(ms > 0 for _, ms in recs), recs
    # a trace that was not restarted records nothing more
    blk.forward(X, 1, out)
    torch.cuda.synchronize()
    assert len(trace.read()) == len(recs)
