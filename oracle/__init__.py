"""CPU oracle for the speculative-decoding verify step.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import or call this package.  The product
path (the CUDA library and its Python binding) never imports it and has no
CPU fallback.  The oracle shares no code with the CUDA path: it is a plain,
slow restatement of what the verify step computes, in numpy float64 with
rounding to bfloat16 / binary32 only where the model stores values in those
formats.
"""
from .verify import *  # noqa: F401,F403
