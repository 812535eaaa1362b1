"""Seeded synthetic inputs for the verify-step workloads.

This subpackage serves both the CUDA path and the CPU oracle.  It draws
numbers (weights, context keys/values, token ids, the uniform draws that
decide drafts) and lays out pages; it holds none of the verify step's
arithmetic (no RoPE, attention, projection or argmax).

The generator itself is C (``specgen.c``, counter-based SplitMix64 plus
Box-Muller); this module compiles it on first use with gcc and calls it
through ctypes.
"""
from .gen import (  # noqa: F401
    fnv1a64,
    normal_bf16,
    normal_bf16_rows,
    normal_f32,
    randint,
    raw_u64,
    uniform,
    generator_threads,
)
from .workloads import WORKLOADS, LayerSpec, Workload, get_workload  # noqa: F401
