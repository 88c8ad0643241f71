"""Where the bf16 error of the scan and of the block comes from, on the CPU (no GPU needed).

For each case four errors are compared, all against the fp64 oracle:
  (i)   only the output rounded to bf16;
  (ii)  the storage floor: the oracle with every tensor a bf16 block stores rounded to bf16 (inputs and
        weights, review tokens, x / B / C / q / k / v, y, O and the output) and nothing else;
  (iii) (ii) plus the tensor-core scan's own rounding points, as first built (bf16 G, bf16 weighted
        inputs of the chunk states, bf16 chunk and carried states);
  (iv)  (ii) plus the scan's rounding points as it now runs on bf16 x (fp16 G and weighted inputs, fp32
        chunk states, carried states as a bf16 hi + lo pair, bf16 intra-chunk operand M);
  (v)   the block as it now runs: (iv) with the projected x stored in fp16 instead of bf16 and M an fp16
        operand (block cases only; the standalone scan takes bf16 x).
The GPU tests bound the measured error by max(2e-2, 1.5 x (ii)); these tests show that the kernel's own
rounding points, (iv), stay inside that bound with room to spare, which (iii) did not.  Scan errors are
element-wise (|g - o| / max(|o|, rms(o))), block errors RMS-normalised (max|g - o| / rms(o))."""
import numpy as np
import pytest

from helpers import BF16_REL, BF16_RMS_ABS, oracle_cached
from bf16_floor import (bf16_storage_forward, elementwise_err, rms_normalised_max_err, round_bf16,
                        rounding_emulation_forward, ssd_rounding_emulation)
import mate_inputs as mi
from edge_configs import all_test_configs
from oracle import mate_oracle as O

SCAN_NAMES = ["bf16_small_8x16x16", "bf16_ragged_12x16x24", "bf16_b2_20x16x16_d512", "bf16_onechunk_4x8x8",
              "bf16_noreview_b2_8x16x16"]


def _scan_inputs(cfg, long_memory, seed=7):
    # the inputs of the GPU scan tests (test_gpu_parity._ssd_inputs)
    rng = np.random.default_rng(seed)
    L = cfg.R + cfg.n
    x = mi.round_to_bf16(rng.standard_normal((cfg.B, L, cfg.nh * cfg.P)))
    Bm = mi.round_to_bf16(rng.standard_normal((cfg.B, L, cfg.N)))
    Cm = mi.round_to_bf16(rng.standard_normal((cfg.B, L, cfg.N)))
    dt = rng.standard_normal((cfg.B, L, cfg.nh)).astype(np.float32)
    dt_bias = np.full(cfg.nh, -4.0 if long_memory else 0.0, np.float32)
    A_log = rng.uniform(-3.0, -1.0, cfg.nh).astype(np.float32) if long_memory else \
        rng.uniform(0.0, 1.0, cfg.nh).astype(np.float32)
    D = rng.standard_normal(cfg.nh).astype(np.float32)
    return x, Bm, Cm, dt, dt_bias, A_log, D


def scan_decomposition(name, long_memory):
    """[(i) = (ii), (iii), (iv)] element-wise errors of the scan entry point's output."""
    cfg = all_test_configs()[name]
    x, Bm, Cm, dt, dt_bias, A_log, D = _scan_inputs(cfg, long_memory)

    def compute():
        ref, emu = [], {"bf16_states": [], "kernel": []}
        for b in range(cfg.B):
            delta = O.softplus(dt[b].astype(np.float64) + dt_bias.astype(np.float64))
            A = -np.exp(A_log.astype(np.float64))
            xs = x[b].astype(np.float64).reshape(-1, cfg.nh, cfg.P)
            args = (xs, Bm[b].astype(np.float64), Cm[b].astype(np.float64), delta, A, D.astype(np.float64), cfg.R)
            ref.append(O.ssd_bidirectional(*args))
            for k in emu:
                emu[k].append(ssd_rounding_emulation(*args, cfg.Q, k))
        ref = np.stack(ref)
        return np.array([elementwise_err(round_bf16(ref), ref)] +
                        [elementwise_err(np.stack(emu[k]), ref) for k in ("bf16_states", "kernel")])
    return oracle_cached(f"floor-decomp-ssd-{name}-{long_memory}", compute)


def block_decomposition(name, layer, variant):
    """[(i), (ii), (iii), (iv), (v)] RMS-normalised errors of the block output."""
    cfg = all_test_configs()[name]
    kw = dict(dt_bias=-4.0, a_log_range=(-3.0, -1.0)) if variant == "long" else {}
    w = mi.make_inputs(cfg, **kw)

    def compute():
        ref = O.mate_forward(w["X"], w, cfg, layer)
        return np.array([rms_normalised_max_err(round_bf16(ref), ref),
                         rms_normalised_max_err(bf16_storage_forward(w["X"], w, cfg, layer), ref)] +
                        [rms_normalised_max_err(rounding_emulation_forward(w["X"], w, cfg, layer, k), ref)
                         for k in ("bf16_states", "kernel", "kernel_f16x")])
    return oracle_cached(f"floor-decomp-mate-{name}-{layer}-{variant}", compute)


@pytest.mark.parametrize("long_memory", [False, True])
@pytest.mark.parametrize("name", SCAN_NAMES)
def test_scan_rounding_points_stay_inside_the_storage_bound(name, long_memory):
    storage, first, now = scan_decomposition(name, long_memory)
    bound = max(BF16_REL, 1.5 * storage)
    print(f"scan {name} long={long_memory}: (i)=(ii) {storage:.3e}  (iii) {first:.3e}  (iv) {now:.3e}  "
          f"bound {bound:.3e}")
    # rounding the output alone is the storage floor here (the scan's inputs are bf16 already): 2^-8
    # relative at most
    assert storage <= 2.0 ** -8
    # the kernel's own rounding points leave a fifth of the bound to accumulation order
    assert now <= 0.8 * bound, (name, long_memory, now, bound)


BLOCK_CASES = [("bf16_small_8x16x16", 0, "default"), ("bf16_small_8x16x16", 3, "default"),
               ("bf16_small_8x16x16", 1, "long"), ("bf16_small_8x16x16", 2, "long"),
               ("bf16_ragged_12x16x24", 1, "long"), ("bf16_noreview_b2_8x16x16", 2, "long")]


@pytest.mark.parametrize("name,layer,variant", BLOCK_CASES)
def test_block_rounding_points_stay_inside_the_storage_bound(name, layer, variant):
    out_only, storage, first, now, block = block_decomposition(name, layer, variant)
    bound = max(BF16_RMS_ABS, 1.5 * storage)
    print(f"block {name} layer {layer} {variant}: (i) {out_only:.3e}  (ii) {storage:.3e}  (iii) {first:.3e}  "
          f"(iv) {now:.3e}  (v) {block:.3e}  bound {bound:.3e}")
    assert out_only <= storage * 1.0001 + 1e-12 or out_only <= 2.0 ** -8 * 20
    assert now <= 0.85 * bound and block <= 0.85 * bound, (name, layer, variant, now, block, bound)
