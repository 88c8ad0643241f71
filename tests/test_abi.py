"""The C ABI library: it builds, loads without a GPU, exports every symbol include/mate.h declares, and
validates arguments on the host before touching the device."""
import ctypes
import dataclasses
import os
import re

import pytest

from helpers import ROOT
from linear_complexity_video_mate_b200 import _lib, build
import mate_inputs as mi


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _header_symbols():
    with open(os.path.join(ROOT, "include", "mate.h")) as f:
        text = f.read()
    return set(re.findall(r"MATE_API\s+[\w\s\*]+?\b(\w+)\s*\(", text))


def test_exports_every_declared_symbol(lib):
    declared = _header_symbols()
    assert declared == set(_lib.EXPORTS), declared ^ set(_lib.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(8):
        assert _lib.status_str(s)


def test_all_workloads_are_valid(lib):
    for name, cfg in mi.all_configs().items():
        c = _lib.make_config(cfg)
        assert lib.mate_check_config(ctypes.byref(c)) == _lib.MATE_OK, name
        assert lib.mate_workspace_bytes(ctypes.byref(c)) > 0, name


def _cfg(**kw):
    base = mi.CONFIGS["bf16_16x32x32"]
    import dataclasses
    return _lib.make_config(dataclasses.replace(base, **kw))


@pytest.mark.parametrize("kw,status", [
    (dict(T=15), _lib.MATE_ERR_SHAPE),            # window does not divide T
    (dict(R=24), _lib.MATE_ERR_SHAPE),            # R not a multiple of 16
    (dict(R=16 * 5), _lib.MATE_ERR_SHAPE),        # pooled grid 5 x 4 x 4 does not divide T = 16
    (dict(st=4), _lib.MATE_ERR_SHAPE),            # shift not smaller than the window
    (dict(P=32), _lib.MATE_ERR_UNSUPPORTED),      # bf16 tensor-core scan needs P = 64
    (dict(tp=64), _lib.MATE_ERR_UNSUPPORTED),
    (dict(d=1004), _lib.MATE_ERR_SHAPE),          # rows not a multiple of 16 bytes
    (dict(d=1000), _lib.MATE_ERR_UNSUPPORTED),    # bf16 projections need d % 64 == 0
    (dict(B=0), _lib.MATE_ERR_SHAPE),
])
def test_config_rejections(lib, kw, status):
    c = _cfg(**kw)
    assert lib.mate_check_config(ctypes.byref(c)) == status
    assert lib.mate_workspace_bytes(ctypes.byref(c)) == 0


def test_null_and_misaligned_arguments_are_rejected_before_launch(lib):
    c = _cfg()
    fake = ctypes.c_void_p(1 << 20)      # aligned, never dereferenced: validation fails first
    mis = ctypes.c_void_p((1 << 20) + 4)
    w = _lib.CWeights(*([1 << 20] * 7))
    cp = ctypes.byref(c)
    assert lib.rms_permute(None, fake, 0, cp, None) == _lib.MATE_ERR_ARG
    assert lib.rms_permute(fake, fake, 4, cp, None) == _lib.MATE_ERR_ARG
    assert lib.rms_unpermute(mis, fake, 1, cp, None) == _lib.MATE_ERR_ARG
    assert lib.review_pool(fake, None, 0, cp, None) == _lib.MATE_ERR_ARG
    assert lib.tesa_forward(fake, None, 1, cp, None) == _lib.MATE_ERR_ARG
    assert lib.mate_forward(fake, ctypes.byref(w), -1, fake, cp, fake, 1 << 40, None) == _lib.MATE_ERR_ARG
    assert lib.mate_forward(fake, None, 0, fake, cp, fake, 1 << 40, None) == _lib.MATE_ERR_ARG
    need = lib.mate_workspace_bytes(cp)
    assert lib.mate_forward(fake, ctypes.byref(w), 0, fake, cp, fake, need - 1, None) == _lib.MATE_ERR_WORKSPACE
    assert lib.ssd_scan_bidir(fake, fake, fake, fake, fake, fake, fake, -1, fake, cp, fake, 1 << 40, None) == \
        _lib.MATE_ERR_ARG
    nss = lib.mate_ssd_workspace_bytes(cp, 256)
    assert lib.ssd_scan_bidir(fake, fake, fake, fake, fake, fake, fake, 256, fake, cp, fake, nss - 1, None) == \
        _lib.MATE_ERR_WORKSPACE
    # Mamba2 extras: the flag is 0 or 1, and with it the four extra weights are required
    ce = _cfg()
    ce.mamba_extras = 2
    assert lib.mate_check_config(ctypes.byref(ce)) == _lib.MATE_ERR_ARG
    ce.mamba_extras = 1
    assert lib.mate_check_config(ctypes.byref(ce)) == _lib.MATE_OK
    assert lib.mate_workspace_bytes(ctypes.byref(ce)) > lib.mate_workspace_bytes(cp)
    assert lib.mate_forward(fake, ctypes.byref(w), 0, fake, ctypes.byref(ce), fake, 1 << 40, None) == \
        _lib.MATE_ERR_ARG
    we = _lib.CWeights(*([1 << 20] * 14))
    we.conv_w = (1 << 20) + 4    # the taps are read as 16-byte vectors
    assert lib.mate_forward(fake, ctypes.byref(we), 0, fake, ctypes.byref(ce), fake, 1 << 40, None) == \
        _lib.MATE_ERR_ARG
    # the timeout self-test takes a bounded poll count
    assert lib.mate_selftest_wait_timeout(0, None) == _lib.MATE_ERR_ARG
    assert lib.mate_selftest_wait_timeout(65537, None) == _lib.MATE_ERR_ARG
    # backward scan: fp32 blocks only, every pointer required, workspace checked
    nbw = lib.mate_ssd_backward_workspace_bytes(cp, 256)
    assert nbw > 0
    bargs = [fake] * 7 + [256] + [fake] * 8
    assert lib.ssd_scan_bidir_backward(*bargs, cp, fake, nbw, None) == _lib.MATE_ERR_UNSUPPORTED   # bf16 config
    cf = _lib.make_config(mi.CONFIGS["tiny_f32_4x8x8"])
    nbf = lib.mate_ssd_backward_workspace_bytes(ctypes.byref(cf), 256)
    assert nbf > 0
    assert lib.ssd_scan_bidir_backward(*bargs, ctypes.byref(cf), fake, nbf - 1, None) == _lib.MATE_ERR_WORKSPACE
    nullargs = list(bargs)
    nullargs[9] = None
    assert lib.ssd_scan_bidir_backward(*nullargs, ctypes.byref(cf), fake, nbf, None) == _lib.MATE_ERR_ARG
    # separate backward-scan parameters: all three or none
    wp = _lib.CWeights(*([1 << 20] * 8))
    assert lib.mate_forward(fake, ctypes.byref(wp), 0, fake, cp, fake, 1 << 40, None) == _lib.MATE_ERR_ARG
    assert lib.ssd_scan_bidir_pd(fake, fake, fake, fake, fake, fake, fake, fake, None, fake, 256, fake, cp, fake,
                                 1 << 40, None) == _lib.MATE_ERR_ARG
    npd = lib.mate_ssd_pd_workspace_bytes(cp, 256)
    assert npd > nss   # the backward scan's own step sizes, decays and review states
    assert lib.ssd_scan_bidir_pd(fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, 256, fake, cp, fake,
                                 npd - 1, None) == _lib.MATE_ERR_WORKSPACE
    assert lib.mate_project_bf16(fake, 512, 128, 1024, fake, 1024, 256, fake, 256, None) == _lib.MATE_ERR_ARG
    assert lib.mate_project_bf16(fake, 1000, 128, 1000, fake, 1000, 256, fake, 256, None) == \
        _lib.MATE_ERR_UNSUPPORTED
    bad = _cfg(T=15)
    assert lib.mate_forward(fake, ctypes.byref(w), 0, fake, ctypes.byref(bad), fake, 1 << 40, None) == \
        _lib.MATE_ERR_SHAPE


def test_workspace_grows_linearly_with_tokens(lib):
    sizes = []
    for T in (16, 64, 256):
        c = _cfg(T=T, R=256)
        sizes.append(lib.mate_workspace_bytes(ctypes.byref(c)))
    per = [(sizes[i + 1] - sizes[i]) for i in range(2)]
    # doubling-by-4 of T adds 4x the per-token bytes each time
    assert abs(per[1] / per[0] - 4.0) < 0.01


def test_noalloc_scan_rejects_problems_beyond_its_scratch(lib):
    """The fixed-scratch scan refuses, before touching the device, a problem whose scratch exceeds the buffer."""
    cfg = mi.CONFIGS["bf16_16x32x32"]
    c = _lib.make_config(cfg)
    assert lib.mate_ssd_workspace_bytes(ctypes.byref(c), cfg.R) > _lib.MATE_SSD_NOALLOC_SCRATCH_BYTES
    st = lib.ssd_scan_bidir_noalloc(16, 16, 16, 16, 16, 16, 16, cfg.R, 16, ctypes.byref(c), None)
    assert st == _lib.MATE_ERR_TOO_LARGE, _lib.status_str(st)


def test_noalloc_scan_limit_follows_the_workspace_size(lib):
    """Shapes on either side of the scratch size: those whose workspace fits are accepted up to the pointer
    check (a null x gives MATE_ERR_ARG, before any device work), the others get MATE_ERR_TOO_LARGE."""
    base = mi.TEST_CONFIGS["bf16_small_8x16x16"]
    seen = set()
    for T in (44, 48, 52, 56, 60):
        cfg = dataclasses.replace(base, T=T, H=8, W=16, R=64)
        c = _lib.make_config(cfg)
        assert lib.mate_check_config(ctypes.byref(c)) == _lib.MATE_OK
        fits = lib.mate_ssd_workspace_bytes(ctypes.byref(c), cfg.R) <= _lib.MATE_SSD_NOALLOC_SCRATCH_BYTES
        seen.add(fits)
        st = lib.ssd_scan_bidir_noalloc(None, 16, 16, 16, 16, 16, 16, cfg.R, 16, ctypes.byref(c), None)
        assert st == (_lib.MATE_ERR_ARG if fits else _lib.MATE_ERR_TOO_LARGE), (T, _lib.status_str(st))
    assert seen == {True, False}


def test_kernel_names_are_distinct(lib):
    names = [lib.mate_kernel_name(k).decode() for k in range(21)]
    assert len(set(names)) == 21 and "unknown" not in names, names
    assert lib.mate_kernel_name(99).decode() == "unknown"
    assert lib.mate_trace_start(-1) == _lib.MATE_ERR_ARG


def test_scan_locality_argument_checks(lib):
    """Rejected before any device work: bad map, null or misaligned output, Hilbert on a grid it does not tile."""
    assert lib.mate_scan_locality(4, 8, 8, 7, 64, None) == _lib.MATE_ERR_ARG
    assert lib.mate_scan_locality(4, 8, 8, 0, None, None) == _lib.MATE_ERR_ARG
    assert lib.mate_scan_locality(4, 8, 8, 0, 68, None) == _lib.MATE_ERR_ARG
    assert lib.mate_scan_locality(0, 8, 8, 0, 64, None) == _lib.MATE_ERR_ARG
    assert lib.mate_scan_locality(64, 48, 48, 5, 64, None) == _lib.MATE_ERR_UNSUPPORTED   # 48 is not a power of two
    assert lib.mate_scan_locality(12, 8, 8, 5, 64, None) == _lib.MATE_ERR_UNSUPPORTED     # 8 does not divide 12
    assert lib.mate_scan_locality(8, 8, 4, 5, 64, None) == _lib.MATE_ERR_UNSUPPORTED      # H != W


def test_plain_c_consumer_compiles_links_and_validates(tmp_path):
    """include/mate.h compiles as C99 and libmate.so links into a plain C program whose host-side checks
    answer as the header states (tests/c_abi_check.c; no device needed)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.dirname(_lib.LIB_PATH)
    exe = str(tmp_path / "c_abi_check")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"),
                    os.path.join(root, "tests", "c_abi_check.c"), "-L", pkg, "-lmate", f"-Wl,-rpath,{pkg}",
                    "-o", exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.startswith("ok"), (r.returncode, r.stdout, r.stderr)
