"""fp64 CPU oracle of gated block-sparse decode attention.

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package. The CUDA library never does.
"""
