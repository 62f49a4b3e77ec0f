"""fp64 CPU oracle for block-sparse video attention (test infrastructure
only: imported by the tests, the smoke check and the benchmark's CPU
baseline, never by the product package)."""
