"""Edge-case block shapes of the GPU tests (kept out of mate_inputs.py, whose digest keys the cached oracle
results): a grid that is exactly one scan chunk and one attention window (its shifted layers mask every
region pair inside the single window), and a batch of two without review tokens."""
import mate_inputs as mi

EDGE_CONFIGS = {
    "bf16_onechunk_4x8x8": mi._cfg("bf16_onechunk_4x8x8", 1, 4, 8, 8, 512, 8, 64, 128, 256, 16, 4, 128, (4, 8, 8),
                                   "bf16", 15),
    "bf16_noreview_b2_8x16x16": mi._cfg("bf16_noreview_b2_8x16x16", 2, 8, 16, 16, 512, 8, 64, 128, 256, 0, 4, 128,
                                        (4, 8, 8), "bf16", 16),
}


def all_test_configs():
    out = mi.all_configs()
    out.update(EDGE_CONFIGS)
    return out
