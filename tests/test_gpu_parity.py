"""Parity of the CUDA library (through the C ABI) with the fp64 oracle, element by element, on seeded
synthetic inputs.  Permutations are compared bit for bit; floating point within the block's tolerances
(helpers.assert_close)."""
import numpy as np
import pytest

from helpers import assert_close, assert_close_elementwise, oracle_cached, requires_gpu
from bf16_floor import bf16_storage_forward, elementwise_err, rms_normalised_max_err, round_bf16
import mate_inputs as mi
from edge_configs import all_test_configs
from oracle import mate_oracle as O

pytestmark = [pytest.mark.gpu, requires_gpu]

torch = pytest.importorskip("torch")
from linear_complexity_video_mate_b200 import mate as M  # noqa: E402


def dev(a, dtype):
    return torch.as_tensor(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def host(t):
    return t.float().cpu().numpy()


def tdt(cfg):
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def cast(cfg, a):
    return mi.round_to_bf16(a) if cfg.dtype == "bf16" else np.asarray(a, np.float32)


SMALL = ["tiny_f32_4x8x8", "f32_b2_4x8x12", "bf16_small_8x16x16", "bf16_ragged_12x16x24", "bf16_b2_20x16x16_d512",
         "bf16_onechunk_4x8x8", "bf16_noreview_b2_8x16x16"]


# ------------------------------------------------------------------ Rotary Major Scan + review tokens

@pytest.mark.parametrize("name", SMALL + ["bf16_16x32x32", "bf16_256x32x32", "bf16_2x64x48x48_d2048"])
def test_rms_permute_unpermute_bitexact(name):
    cfg = all_test_configs()[name]
    X = mi.make_x_only(cfg, 100)
    Xd = dev(X, tdt(cfg))
    for order in range(4):
        Xp = M.rms_permute(Xd, order, cfg)
        torch.cuda.synchronize()
        got = host(Xp)
        for b in range(cfg.B):
            pos = O.scan_positions(cfg.T, cfg.H, cfg.W, order).ravel()
            expect = np.empty((cfg.n, cfg.d), np.float32)
            expect[pos] = X[b].reshape(cfg.n, cfg.d)        # row s(t,h,w) = X[t,h,w]
            assert np.array_equal(got[b], expect), (name, order, b)
        back = M.rms_unpermute(Xp, order, cfg)
        assert torch.equal(back, Xd), (name, order)


@pytest.mark.parametrize("name", SMALL + ["bf16_256x32x32"])
def test_review_pool(name):
    cfg = all_test_configs()[name]
    X = mi.make_x_only(cfg, 101)
    Xd = dev(X, tdt(cfg))
    for order in range(4):
        got = host(M.review_pool(Xd, order, cfg))
        ref = np.stack([O.review_tokens(X[b], cfg.R, order) for b in range(cfg.B)])
        if cfg.dtype == "bf16":
            # fp32 accumulation then one bf16 rounding: within one bf16 unit of the exact mean
            assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6), (name, order)
        else:
            np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-6)


# ------------------------------------------------------------------ tensor-core projection

@pytest.mark.parametrize("M_,K,N", [(128, 64, 128), (300, 1024, 4368), (1024, 2048, 1024), (77, 512, 2336),
                                    (4096, 1024, 8480)])
def test_project_bf16(M_, K, N):
    rng = np.random.default_rng(M_ + K + N)
    A = mi.round_to_bf16(rng.standard_normal((M_, K)))
    W = mi.round_to_bf16(rng.standard_normal((N, K)) / np.sqrt(K))
    got = host(M.project_bf16(dev(A, torch.bfloat16), dev(W, torch.bfloat16)))
    ref = A.astype(np.float64) @ W.astype(np.float64).T
    assert_close(got, ref, "bf16", f"project {M_}x{K}x{N}")


# ------------------------------------------------------------------ selective scan

def _ssd_inputs(cfg, long_memory, seed):
    rng = np.random.default_rng(seed)
    L = cfg.R + cfg.n
    x = cast(cfg, rng.standard_normal((cfg.B, L, cfg.nh * cfg.P)))
    Bm = cast(cfg, rng.standard_normal((cfg.B, L, cfg.N)))
    Cm = cast(cfg, rng.standard_normal((cfg.B, L, cfg.N)))
    dt = rng.standard_normal((cfg.B, L, cfg.nh)).astype(np.float32)
    dt_bias = np.full(cfg.nh, -4.0 if long_memory else 0.0, np.float32)
    A_log = rng.uniform(-3.0, -1.0, cfg.nh).astype(np.float32) if long_memory else \
        rng.uniform(0.0, 1.0, cfg.nh).astype(np.float32)
    D = rng.standard_normal(cfg.nh).astype(np.float32)
    return x, Bm, Cm, dt, dt_bias, A_log, D


def _ssd_oracle(cfg, x, Bm, Cm, dt, dt_bias, A_log, D, heads=None):
    heads = list(range(cfg.nh)) if heads is None else heads
    out = []
    for b in range(cfg.B):
        xs = x[b].reshape(-1, cfg.nh, cfg.P)[:, heads]
        delta = O.softplus(dt[b].astype(np.float64) + dt_bias.astype(np.float64))[:, heads]
        A = -np.exp(A_log.astype(np.float64))[heads]
        out.append(O.ssd_bidirectional(xs, Bm[b], Cm[b], delta, A, D.astype(np.float64)[heads], cfg.R))
    return np.stack(out)   # [B, n, len(heads), P]


@pytest.mark.parametrize("long_memory", [False, True])
@pytest.mark.parametrize("name", SMALL)
def test_ssd_scan_bidir(name, long_memory):
    cfg = all_test_configs()[name]
    args = _ssd_inputs(cfg, long_memory, 7)
    x, Bm, Cm, dt, dt_bias, A_log, D = args
    td = tdt(cfg)
    y = M.ssd_scan_bidir(dev(x, td), dev(Bm, td), dev(Cm, td), dev(dt, torch.float32), dev(dt_bias, torch.float32),
                         dev(A_log, torch.float32), dev(D, torch.float32), cfg.R, cfg)
    got = host(y).reshape(cfg.B, cfg.n, cfg.nh, cfg.P)
    ref = oracle_cached(f"ssd-{name}-{long_memory}", lambda: _ssd_oracle(cfg, *args))
    assert_close_elementwise(got, ref, cfg.dtype, f"ssd {name} long={long_memory}", _ssd_floor(cfg, ref))


@pytest.mark.parametrize("regime", ["fast_decay", "no_decay"])
@pytest.mark.parametrize("name", ["tiny_f32_4x8x8", "bf16_small_8x16x16", "bf16_noreview_b2_8x16x16"])
def test_ssd_scan_extreme_decays(name, regime):
    """Degenerate step sizes and decays.  fast_decay: delta A below -80 per token, every decay underflows
    and y reduces to the diagonal 2 (D + C_i . B_i delta_i) x_i.  no_decay: A about -1e-13 with small steps,
    so the states are plain running sums over the whole sequence (both carries at full weight)."""
    cfg = all_test_configs()[name]
    x, Bm, Cm, dt, dt_bias, A_log, D = _ssd_inputs(cfg, False, 17)
    if regime == "fast_decay":
        A_log = np.full(cfg.nh, 7.0, np.float32)
        dt_bias = np.full(cfg.nh, 2.0, np.float32)
    else:
        A_log = np.full(cfg.nh, -30.0, np.float32)
        dt_bias = np.full(cfg.nh, -6.0, np.float32)
    args = (x, Bm, Cm, dt, dt_bias, A_log, D)
    td = tdt(cfg)
    y = M.ssd_scan_bidir(dev(x, td), dev(Bm, td), dev(Cm, td), dev(dt, torch.float32), dev(dt_bias, torch.float32),
                         dev(A_log, torch.float32), dev(D, torch.float32), cfg.R, cfg)
    got = host(y).reshape(cfg.B, cfg.n, cfg.nh, cfg.P)
    key = f"ssd-{name}-{regime}"
    ref = oracle_cached(key, lambda: _ssd_oracle(cfg, *args))
    if regime == "fast_decay":   # the closed form of the degenerate case pins the oracle too
        delta = O.softplus(dt.astype(np.float64) + 2.0)[:, cfg.R:]
        cb = np.einsum("bln,bln->bl", Cm.astype(np.float64), Bm.astype(np.float64))[:, cfg.R:]
        diag = 2.0 * (D[None, None, :] + cb[:, :, None] * delta)
        want = diag[..., None] * x.astype(np.float64)[:, cfg.R:].reshape(cfg.B, cfg.n, cfg.nh, cfg.P)
        # (a large cached oracle result is stored in float16, relative 2^-11: a bound of 2^-10 is still far
        # below any dropped term, which would move values by a relative O(1))
        assert np.abs(ref - want).max() <= 2.0 ** -10 * max(1.0, np.abs(want).max())
    assert_close_elementwise(got, ref, cfg.dtype, f"ssd {name} {regime}", _ssd_floor(cfg, ref))


def _ssd_floor(cfg, ref):
    """Storage floor of the scan entry point (0 for fp32 blocks): its inputs are bf16 already, so its only
    stored bf16 tensor is the output y; the element-wise error of bf16(ref) against ref."""
    if cfg.dtype != "bf16":
        return 0.0
    return elementwise_err(round_bf16(ref), ref)


# ------------------------------------------------------------------ TESA

def _tesa_inputs(cfg, seed):
    rng = np.random.default_rng(seed)
    return cast(cfg, rng.standard_normal((cfg.B, cfg.T, cfg.H, cfg.W, 3 * cfg.th * cfg.tp)))


@pytest.mark.parametrize("shifted", [False, True])
@pytest.mark.parametrize("name", SMALL + ["bf16_16x32x32"])
def test_tesa_forward(name, shifted):
    cfg = all_test_configs()[name]
    qkv = _tesa_inputs(cfg, 8)
    got = host(M.tesa_forward(dev(qkv, tdt(cfg)), shifted, cfg))
    ref = oracle_cached(f"tesa-{name}-{shifted}", lambda: np.stack([
        O.tesa_attention(qkv[b], cfg.th, cfg.tp, (cfg.wt, cfg.wh, cfg.ww), (cfg.st, cfg.sh, cfg.sw), shifted)
        for b in range(cfg.B)]))
    assert_close_elementwise(got, ref, cfg.dtype, f"tesa {name} shifted={shifted}")


# ------------------------------------------------------------------ whole block

def _sample_rows(cfg, k=4096, seed=5, keep_every=4):
    """A fixed random subset of the block's output rows (all rows when the block has at most k): every
    keep_every-th of k sorted random rows, i.e. 1024 rows spread over the whole block."""
    rows = cfg.B * cfg.n
    if rows <= k:
        return np.arange(rows)
    return np.sort(np.random.default_rng(seed).choice(rows, size=k, replace=False))[::keep_every]


def _block(cfg, variant):
    kw = dict(dt_bias=-4.0, a_log_range=(-3.0, -1.0)) if variant == "long" else {}
    return mi.make_inputs(cfg, **kw)


def block_reference(cfg, w, layer, variant):
    """(rows, oracle output on those rows, bf16 storage floor on them) of a block case: all rows of a small
    block, or a fixed sample of 1024 rows of a large one (whose oracle output is cached only on those
    rows)."""
    rows = _sample_rows(cfg)
    key = f"{cfg.name}-{layer}-{variant}" + ("" if len(rows) == cfg.B * cfg.n else f"-rows{len(rows)}")
    holder = {}

    def full():
        if "ref" not in holder:
            holder["ref"] = O.mate_forward(w["X"], w, cfg, layer).reshape(cfg.B * cfg.n, cfg.d)
        return holder["ref"]

    ref = oracle_cached(f"mate-{key}", lambda: full()[rows]).reshape(len(rows), cfg.d)
    floor = 0.0
    if cfg.dtype == "bf16":
        floor = float(oracle_cached(f"floor-{key}", lambda: np.array([rms_normalised_max_err(
            bf16_storage_forward(w["X"], w, cfg, layer).reshape(cfg.B * cfg.n, cfg.d)[rows], ref)]))[0])
    return rows, ref, floor


def _check_block(cfg, w, layer, variant, out):
    """Compare the GPU block output with the oracle (see block_reference)."""
    rows, ref, floor = block_reference(cfg, w, layer, variant)
    got = np.asarray(out).reshape(cfg.B * cfg.n, cfg.d)[rows]
    assert_close(got, ref, cfg.dtype, f"mate {cfg.name} layer {layer} {variant}", floor)


@pytest.mark.parametrize("variant", ["default", "long"])
@pytest.mark.parametrize("layer", [0, 1, 2, 3])
@pytest.mark.parametrize("name", SMALL + ["bf16_16x32x32"])
def test_mate_forward(name, layer, variant):
    cfg = all_test_configs()[name]
    w = _block(cfg, variant)
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    out = host(blk.forward(dev(w["X"], tdt(cfg)), layer))
    _check_block(cfg, w, layer, variant, out)


@pytest.mark.parametrize("layer", [0, 1, 2, 3])
@pytest.mark.parametrize("branch", ["te", "ma"])
@pytest.mark.parametrize("name", ["bf16_small_8x16x16", "bf16_ragged_12x16x24", "bf16_b2_20x16x16_d512"])
def test_mate_forward_single_branch(name, branch, layer):
    """Each branch alone (the other branch's output projection zeroed).  The TE branch's output is not
    heavy-tailed, so its bf16-storage floor stays below 2e-2 and the strict bound applies."""
    cfg = all_test_configs()[name]
    w = dict(_block(cfg, "default"))
    zero = "W_out" if branch == "te" else "W_o"
    w[zero] = np.zeros_like(w[zero])
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    out = host(blk.forward(dev(w["X"], tdt(cfg)), layer))
    _check_block(cfg, w, layer, f"{branch}only", out)


@pytest.mark.parametrize("name,layer", [("bf16_small_8x16x16", 3), ("bf16_b2_20x16x16_d512", 2),
                                        ("bf16_onechunk_4x8x8", 1), ("bf16_noreview_b2_8x16x16", 0)])
def test_mate_forward_host_matches_device_path(name, layer):
    """Host buffers (row-chunked copies overlapped with the projections, including chunks that are empty or
    cross a sample boundary) give the same bits as the device-buffer call."""
    cfg = all_test_configs()[name]
    w = _block(cfg, "default")
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    Xd = dev(w["X"], torch.bfloat16)
    ref = blk.forward(Xd, layer)
    xh = Xd.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    blk.forward_host(xh, layer, oh)
    torch.cuda.synchronize()
    assert torch.equal(oh, ref.cpu())


def test_packed_weights_match_per_call_packing():
    """Weights packed once (mate_pack_weights, the default of MateBlock) and packed again inside every call
    give the same bits."""
    cfg = all_test_configs()["bf16_b2_20x16x16_d512"]
    w = _block(cfg, "default")
    wd = M.weights_to_device(w, cfg)
    Xd = dev(w["X"], torch.bfloat16)
    for layer in (1, 2):
        a = M.MateBlock(cfg, wd).forward(Xd, layer)
        b = M.MateBlock(cfg, wd, pack=False).forward(Xd, layer)
        assert torch.equal(a, b), layer


def test_pipelined_host_calls_match_device_path():
    """Pipelined host calls (each input copy overlapping the previous call's output copy, inputs in
    alternating device slots): a chain whose every output is the next call's input (the output copy must
    land before the next input copy reads it), then calls that reuse one input buffer; all bit-equal to
    the device-buffer path."""
    cfg = all_test_configs()["bf16_small_8x16x16"]
    w = dict(_block(cfg, "default"))
    # the MA branch's output grows with the cube of its input, so a chain through it overflows in a few
    # steps; the chain runs the attention branch alone, which is linear in its input
    w["W_out"] = np.zeros_like(w["W_out"])
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    X0 = dev(w["X"], torch.bfloat16)
    dchain = [X0]
    for layer in range(3):
        dchain.append(blk.forward(dchain[-1], layer).clone())
    hchain = [X0.cpu().pin_memory()] + [torch.empty_like(X0, device="cpu").pin_memory() for _ in range(3)]
    for layer in range(3):
        blk.forward_host(hchain[layer], layer, hchain[layer + 1], pipelined=True)
    M.MateBlock.flush_host()
    torch.cuda.synchronize()
    for layer in range(3):
        assert torch.equal(hchain[layer + 1], dchain[layer + 1].cpu()), f"chain step {layer}"
    outs = [torch.empty_like(hchain[0]).pin_memory() for _ in range(4)]
    for layer in range(4):
        blk.forward_host(hchain[0], layer, outs[layer], pipelined=True)
    M.MateBlock.flush_host()
    torch.cuda.synchronize()
    for layer in range(4):
        assert torch.equal(outs[layer], blk.forward(X0, layer).cpu()), f"shared input, layer {layer}"
    assert M.device_status() == 0


def test_repeated_calls_are_deterministic():
    cfg = mi.TEST_CONFIGS["bf16_ragged_12x16x24"]
    w = _block(cfg, "long")
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    Xd = dev(w["X"], torch.bfloat16)
    a = blk.forward(Xd, 1).clone()
    for _ in range(3):
        assert torch.equal(blk.forward(Xd, 1), a)
    assert M.device_status() == 0


# ------------------------------------------------------------------ full-size workloads

# The workloads at full size: all four layers of the 65,536-token clip (every scan order, both shift
# phases), and at the 262,144-token and the batch-2 d = 2048 workloads a spatial-order layer and the two
# time-fastest orders (whose scan output goes through the scan-order buffer), plus the long-memory block.
FULL_SIZE_CASES = [("bf16_64x32x32", 0, "default"), ("bf16_64x32x32", 1, "default"),
                   ("bf16_64x32x32", 2, "default"), ("bf16_64x32x32", 3, "default"),
                   ("bf16_256x32x32", 1, "default"), ("bf16_256x32x32", 2, "default"),
                   ("bf16_256x32x32", 3, "default"), ("bf16_256x32x32", 0, "long"),
                   ("bf16_2x64x48x48_d2048", 1, "default"), ("bf16_2x64x48x48_d2048", 2, "default"),
                   ("bf16_2x64x48x48_d2048", 3, "default")]


@pytest.mark.parametrize("name,layer,variant", FULL_SIZE_CASES)
def test_mate_forward_full_size(name, layer, variant):
    """The block at its full workload sizes, in the launch configuration the benchmark times."""
    cfg = mi.CONFIGS[name]
    w = _block(cfg, variant)
    blk = M.MateBlock(cfg, M.weights_to_device(w, cfg))
    out = host(blk.forward(dev(w["X"], torch.bfloat16), layer))
    del blk
    _check_block(cfg, w, layer, variant, out)


def test_ssd_full_size_sampled_head():
    cfg = mi.CONFIGS["bf16_256x32x32"]
    args = _ssd_inputs(cfg, True, 9)
    x, Bm, Cm, dt, dt_bias, A_log, D = args
    y = M.ssd_scan_bidir(dev(x, torch.bfloat16), dev(Bm, torch.bfloat16), dev(Cm, torch.bfloat16),
                         dev(dt, torch.float32), dev(dt_bias, torch.float32), dev(A_log, torch.float32),
                         dev(D, torch.float32), cfg.R, cfg)
    rows = np.arange(0, cfg.n, 16)   # every 16th video row of head 5: 16384 rows spread over the sequence
    got = host(y).reshape(cfg.B, cfg.n, cfg.nh, cfg.P)[:, rows][:, :, [5]]
    key = "ssd-full-bf16_256x32x32-h5-every16"
    ref = oracle_cached(key, lambda: _ssd_oracle(cfg, *args, heads=[5])[:, rows])
    assert_close_elementwise(got, ref, "bf16", "ssd full size head 5", _ssd_floor(cfg, ref))


# ------------------------------------------------------------------ scan locality

from oracle import scan_locality as SL  # noqa: E402


@pytest.mark.parametrize("grid", [(4, 8, 8), (12, 16, 24), (16, 32, 32), (256, 32, 32), (64, 48, 48)])
@pytest.mark.parametrize("kind", range(7))
def test_scan_locality_exact(grid, kind):
    """Integer sums over all grid-adjacent pairs: bit-exact against the oracle, up to the workload grids."""
    T, H, W = grid
    if kind == 5 and (H != W or H & (H - 1) or T % H):
        pytest.skip("Hilbert map needs H = W a power of two dividing T")
    got = M.scan_locality(T, H, W, kind)
    ref = SL.scan_locality(T, H, W, kind)   # exact integers (not through the float cache)
    assert got == ref, (grid, kind, got, ref)
