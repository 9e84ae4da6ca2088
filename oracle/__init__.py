"""CPU oracle for the ReSA decode hot path.

TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the benchmark's
CPU-baseline leg may import this package; the CUDA library and its Python
binding never do, and the two share no code.
"""
