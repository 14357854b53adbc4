"""Seeded synthetic inputs for the fused int8 GroupedMatmul + MoeFinalizeRouting op.

This package is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark.  It holds only random-number draws and data layout (routing a token to
its experts and sorting the (token, slot) pairs by expert); none of the op's
arithmetic (no matmul, no dequantisation, no combine, no int4 unpacking, no
per-token quantisation) lives here.
"""
from .inputs import CONFIGS, Problem, make_problem, make_routing, sample_rows  # noqa: F401
