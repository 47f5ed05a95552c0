"""Paged-attention oracle: plain CPU reference implementations in fp64.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package.  It shares no code with the CUDA
library and never imports it.
"""
