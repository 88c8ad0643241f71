"""fp64 CPU oracle of the MATE block: test infrastructure only (tests, smoke check, CPU-baseline leg)."""
