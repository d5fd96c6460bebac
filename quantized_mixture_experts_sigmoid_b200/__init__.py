"""Routed Mixture-of-Experts layer for NVIDIA B200 (sm_100a).

The kernels live in libmoe.so behind the C ABI of include/moe.h; ``moe`` is
its Python binding.
"""
from . import moe  # noqa: F401
