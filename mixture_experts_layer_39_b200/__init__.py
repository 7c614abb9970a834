"""Dropless mixture-of-experts expert layer for NVIDIA B200 (sm_100a).

The compute lives in libmoe.so (hand-written CUDA, C ABI in include/moe.h);
this package is its Python binding (ops, MoELayer) plus the seeded
synthetic-input generator (inputs).  Importing the package does not load the
library; the first call does, and fails loudly if it was not built.
"""

__all__ = ["ops", "layer", "inputs", "build"]
