"""fp64 CPU oracle of route-layer chunk-routing sparse attention (test infrastructure).

Only tests/, the smoke check and the benchmark's CPU-baseline leg use this package.
"""
