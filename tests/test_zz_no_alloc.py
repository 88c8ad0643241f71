"""ssd_scan_bidir_noalloc (fixed device scratch, no allocation) against ssd_scan_bidir (caller workspace),
through the C ABI.  Some callers are handed their input and output buffers but may not allocate device
memory themselves (a plugin whose host framework owns every allocation, a serving loop that cannot afford
cudaMalloc's device-wide synchronisation); the no-alloc entry point serves them.

Both entry points run the same kernels on the same inputs, so their outputs must agree bit for bit: a
tolerance could hide a read of scratch bytes left over from an earlier call.  The calls come in a row on
scratch that the previous call left behind (the second call is smaller than the first), and free device
memory is the same before and after a call once the library's device code is loaded.  The file is named
to be collected last, so a run that stops at the first failure has run every other test before it."""
import ctypes

import numpy as np
import pytest

from helpers import requires_gpu
import mate_inputs as mi

pytestmark = [pytest.mark.gpu, requires_gpu]

torch = pytest.importorskip("torch")
from linear_complexity_video_mate_b200 import _lib, mate as M  # noqa: E402

# largest first: the later calls run on scratch that still holds an earlier call's bytes
CASES = (("bf16_b2_20x16x16_d512", 31), ("bf16_small_8x16x16", 32), ("tiny_f32_4x8x8", 33))


def _inputs(cfg, seed):
    rng = np.random.default_rng(seed)
    L = cfg.R + cfg.n
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    act = lambda a: torch.as_tensor(np.asarray(mi.round_to_bf16(a) if cfg.dtype == "bf16" else a, np.float32)).to(
        device="cuda", dtype=tdt)
    f32 = lambda a: torch.as_tensor(np.asarray(a, np.float32)).to(device="cuda")
    return (act(rng.standard_normal((cfg.B, L, cfg.nh * cfg.P))), act(rng.standard_normal((cfg.B, L, cfg.N))),
            act(rng.standard_normal((cfg.B, L, cfg.N))), f32(rng.standard_normal((cfg.B, L, cfg.nh))),
            f32(np.zeros(cfg.nh)), f32(rng.uniform(0.0, 1.0, cfg.nh)), f32(rng.standard_normal(cfg.nh)))


def _noalloc(lib, cfg, c, args, y):
    st = lib.ssd_scan_bidir_noalloc(*[a.data_ptr() for a in args], cfg.R, y.data_ptr(), ctypes.byref(c), None)
    assert st == _lib.MATE_OK, _lib.status_str(st)


def test_noalloc_scan_matches_workspace_scan_on_calls_in_a_row():
    lib = _lib.load()
    cases = []
    for name, seed in CASES:   # every device allocation of the test happens here, before the calls
        cfg = mi.all_configs()[name]
        c = _lib.make_config(cfg)
        assert lib.mate_ssd_workspace_bytes(ctypes.byref(c), cfg.R) <= _lib.MATE_SSD_NOALLOC_SCRATCH_BYTES
        args = _inputs(cfg, seed)
        ref = M.ssd_scan_bidir(*args, cfg.R, cfg)
        y = torch.full((cfg.B, cfg.n, cfg.nh * cfg.P), float("nan"), dtype=args[0].dtype, device="cuda")
        cases.append((name, cfg, c, args, ref, y))
    torch.cuda.synchronize()

    # first call (it may load the library's device code, which holds the scratch array)
    _noalloc(lib, *cases[0][1:4], cases[0][5])
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    # second call, smaller, on the scratch the first one left behind: no device memory is taken
    _noalloc(lib, *cases[1][1:4], cases[1][5])
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    # third call: the fp32 path, whose step sizes also live in the scratch
    _noalloc(lib, *cases[2][1:4], cases[2][5])
    flags = ctypes.c_uint(0)
    assert lib.mate_device_status(None, ctypes.byref(flags)) == _lib.MATE_OK, flags.value

    for name, cfg, c, args, ref, y in cases:
        assert torch.equal(y, ref), f"{name}: no-alloc output differs from the workspace scan"
