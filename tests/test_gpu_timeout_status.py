"""The timeout report of the bounded device waits, exercised on the GPU without a fault: a one-thread
kernel waits on a barrier nothing completes for a bounded number of polls, records a timeout in the
device status word and returns; the host reads MATE_ERR_TIMEOUT once, the word is cleared, and the
context stays usable for ordinary work."""
import ctypes

import numpy as np
import pytest

from helpers import requires_gpu

pytestmark = [pytest.mark.gpu, requires_gpu]

torch = pytest.importorskip("torch")
from linear_complexity_video_mate_b200 import _lib, mate as M  # noqa: E402


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    lib = _lib.load()
    assert M.device_status() == 0                         # clean start (reads and clears the word)
    flags = ctypes.c_uint(0)
    try:
        assert lib.mate_selftest_wait_timeout(1000, None) == _lib.MATE_OK
        first = lib.mate_device_status(None, ctypes.byref(flags))
        got_flags = flags.value
    finally:
        lib.mate_device_status(None, ctypes.byref(flags))  # never leave the word set for later tests
    assert first == _lib.MATE_ERR_TIMEOUT and got_flags & 1, (first, got_flags)
    assert lib.mate_device_status(None, ctypes.byref(flags)) == _lib.MATE_OK and flags.value == 0
    # ordinary work afterwards
    rng = np.random.default_rng(3)
    A = torch.as_tensor(rng.standard_normal((256, 128)), dtype=torch.bfloat16).cuda()
    W = torch.as_tensor(rng.standard_normal((128, 128)) / 11.0, dtype=torch.bfloat16).cuda()
    C = M.project_bf16(A, W).float()
    ref = A.float() @ W.float().T
    assert torch.allclose(C, ref, rtol=2e-2, atol=2e-2 * ref.abs().max().item())
    assert M.device_status() == 0
