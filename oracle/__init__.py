"""Reference oracle for the ternary-weight linear layer — test infrastructure
only (tests, the smoke check and the CPU-baseline leg of the benchmark)."""
