"""Shared test helpers: tolerances, GPU/library availability and a cache of oracle results."""
import hashlib
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CACHE = os.path.join(ROOT, "tests", ".oracle_cache")

# Tolerances of the block (element-wise against the fp64 oracle):
#   fp32 blocks: max|gpu - oracle| / max|oracle| <= 1e-4
#   bf16 blocks: the same ratio <= 2e-2, and max|gpu - oracle| <= 2e-2 after dividing both by the
#   oracle output's RMS.
F32_REL = 1e-4
BF16_REL = 2e-2
BF16_RMS_ABS = 2e-2


def errors(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "non-finite values in the GPU output"
    diff = np.abs(got - ref)
    rel = diff.max() / max(np.abs(ref).max(), 1e-30)
    rms = np.sqrt(np.mean(ref * ref))
    rms_abs = diff.max() / max(rms, 1e-30)
    return rel, rms_abs


# Errors measured by the parity tests, written as JSON lines to the file named by MATE_PARITY_REPORT (if
# set) so that a GPU run leaves the measured column of the error decomposition behind.
_REPORT = os.environ.get("MATE_PARITY_REPORT")


def _report(**kw):
    if _REPORT:
        import json
        with open(_REPORT, "a") as f:
            f.write(json.dumps(kw) + "\n")


def assert_close_elementwise(got, ref, dtype, what="", floor=0.0):
    """Criterion for the intermediate entry points (scan output y, attention output O), whose values are
    heavy-tailed and stored in bf16: bf16 storage alone moves an element by up to 2^-9 of its own
    magnitude, which for max|o| / rms(o) ~ 25 already exceeds 2e-2 * rms(o).  So each element must satisfy
    |g - o| <= tol * max(|o|, rms(o)) with tol = 1e-4 (fp32) or, for bf16, max(2e-2, 1.5 * floor), floor
    being the same error of the oracle's result with only its bf16 storage rounding applied (the storage
    floor, tests/bf16_floor.py; the scan's only stored bf16 tensor is its output); plus the block's
    relative criterion."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape and np.isfinite(got).all()
    tol = max(BF16_REL, 1.5 * floor) if dtype == "bf16" else F32_REL
    rms = np.sqrt(np.mean(ref * ref))
    elem = (np.abs(got - ref) / np.maximum(np.abs(ref), rms)).max()
    rel = np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30)
    rtol = BF16_REL if dtype == "bf16" else F32_REL
    _report(kind="elementwise", what=what, dtype=dtype, elem=float(elem), rel=float(rel), floor=float(floor),
            tol=float(tol))
    assert elem <= tol and rel <= rtol, \
        f"{what}: elementwise err {elem:.3e} (<= {tol:.3e}, bf16 storage floor {floor:.3e}), max rel err {rel:.3e}"
    return elem, rel


def assert_close(got, ref, dtype, what="", floor=0.0):
    """Block-output criterion.  fp32: relative error <= 1e-4.  bf16: relative error <= 2e-2 and
    RMS-normalised max error <= max(2e-2, 1.5 * floor), floor = the same error of the oracle run with bf16
    storage rounding (tests/bf16_floor.py); pass floor = 0 where no floor applies."""
    rel, rms_abs = errors(got, ref)
    _report(kind="block", what=what, dtype=dtype, rel=float(rel), rms_abs=float(rms_abs), floor=float(floor),
            lim=float(max(BF16_RMS_ABS, 1.5 * floor)) if dtype != "f32" else None)
    if dtype == "f32":
        assert rel <= F32_REL, f"{what}: max rel err {rel:.3e} > {F32_REL}"
    else:
        lim = max(BF16_RMS_ABS, 1.5 * floor)
        assert rel <= BF16_REL and rms_abs <= lim, \
            f"{what}: max rel err {rel:.3e} (<= {BF16_REL}), rms-normalised max err {rms_abs:.3e} (<= {lim:.3e}; " \
            f"bf16 storage floor {floor:.3e})"
    return rel, rms_abs


def _code_of(path):
    """What a Python source computes, without its comments and docstrings: edits of the documentation leave
    the cached results valid, any change of the code invalidates them."""
    import ast
    with open(path, "rb") as fh:
        tree = ast.parse(fh.read())
    for node in ast.walk(tree):
        body = getattr(node, "body", None)
        if isinstance(body, list) and body and isinstance(body[0], ast.Expr) and \
                isinstance(getattr(body[0], "value", None), ast.Constant) and isinstance(body[0].value.value, str):
            node.body = body[1:] or [ast.Pass()]
    return ast.dump(tree, include_attributes=False).encode()


def _oracle_digest(extra=()):
    h = hashlib.sha256()
    for f in ("oracle/mate_oracle.py", "mate_inputs.py") + tuple(extra):
        h.update(_code_of(os.path.join(ROOT, f)))
    return h.hexdigest()[:16]


CACHE_BIG = os.path.join(ROOT, ".oracle_cache_big")
BIG_BYTES = 8 << 20


def oracle_cached(key: str, fn, extra=()):
    """fn() -> np.ndarray, cached on disk (see store_dtype: far below every tolerance) under a key that includes
    the oracle's source digest (plus the files `extra` names; keys holding "floor" also digest
    tests/bf16_floor.py, which computes the floors).  Small results and large ones are kept in separate
    folders."""
    if "floor" in key:
        extra = tuple(extra) + ("tests/bf16_floor.py",)
    name = f"{key}-{_oracle_digest(extra)}.npy"
    for d in (CACHE, CACHE_BIG):
        if os.path.exists(os.path.join(d, name)):
            return np.load(os.path.join(d, name)).astype(np.float64)
    out = np.asarray(fn(), dtype=np.float64)
    d = CACHE_BIG if out.size * 4 > BIG_BYTES else CACHE
    os.makedirs(d, exist_ok=True)
    path = os.path.join(d, name)
    np.save(path + ".tmp.npy", out.astype(store_dtype(out)))
    os.replace(path + ".tmp.npy", path)
    return out


def store_dtype(a):
    """Storage type of a cached result: float16 for large arrays (relative rounding 2^-11, forty times below
    the bf16 tolerances; only bf16 test cases produce arrays this large, and finite values below 65504) and
    float32 otherwise (the fp32 test cases' results, compared at 1e-4, are all small)."""
    a = np.asarray(a)
    if a.size > (1 << 18) and np.isfinite(a).all() and np.abs(a).max() < 6e4:
        return np.float16
    return np.float32


def gpu_ready():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


requires_gpu = pytest.mark.skipif(not gpu_ready(), reason="needs a CUDA GPU")
