"""ssd_scan_bidir_noalloc (fixed device scratch, no allocation) against ssd_scan_bidir (caller workspace),
through the C ABI, on two calls in a row.  The second call is smaller than the first, so it runs on scratch
that still holds the first call's contents."""
import ctypes

import numpy as np
import pytest

from helpers import assert_close, requires_gpu
import mate_inputs as mi

pytestmark = [pytest.mark.gpu, requires_gpu]

torch = pytest.importorskip("torch")
from linear_complexity_video_mate_b200 import _lib, mate as M  # noqa: E402


def _inputs(cfg, seed):
    rng = np.random.default_rng(seed)
    L = cfg.R + cfg.n
    bf = lambda a: torch.as_tensor(mi.round_to_bf16(a)).to(device="cuda", dtype=torch.bfloat16)
    f32 = lambda a: torch.as_tensor(np.asarray(a, np.float32)).to(device="cuda")
    return (bf(rng.standard_normal((cfg.B, L, cfg.nh * cfg.P))), bf(rng.standard_normal((cfg.B, L, cfg.N))),
            bf(rng.standard_normal((cfg.B, L, cfg.N))), f32(rng.standard_normal((cfg.B, L, cfg.nh))),
            f32(np.zeros(cfg.nh)), f32(rng.uniform(0.0, 1.0, cfg.nh)), f32(rng.standard_normal(cfg.nh)))


def test_noalloc_scan_matches_workspace_scan_on_two_calls():
    lib = _lib.load()
    for name, seed in (("bf16_b2_20x16x16_d512", 31), ("bf16_small_8x16x16", 32)):
        cfg = mi.all_configs()[name]
        c = _lib.make_config(cfg)
        assert lib.mate_ssd_workspace_bytes(ctypes.byref(c), cfg.R) <= _lib.MATE_SSD_NOALLOC_SCRATCH_BYTES
        args = _inputs(cfg, seed)
        ref = M.ssd_scan_bidir(*args, cfg.R, cfg)
        y = torch.full((cfg.B, cfg.n, cfg.nh * cfg.P), float("nan"), dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()
        st = lib.ssd_scan_bidir_noalloc(*[a.data_ptr() for a in args], cfg.R, y.data_ptr(), ctypes.byref(c), None)
        assert st == _lib.MATE_OK, _lib.status_str(st)
        flags = ctypes.c_uint(0)
        assert lib.mate_device_status(None, ctypes.byref(flags)) == _lib.MATE_OK, flags.value
        got = y.float().cpu().numpy()
        assert np.isfinite(got).all(), name
        assert_close(got, ref.float().cpu().numpy(), "bf16", f"noalloc scan {name}")
