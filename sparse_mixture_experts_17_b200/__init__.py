"""B200-native forward pass of a top-k routed Mixture-of-Experts SwiGLU layer.

`moe` is the Python binding of libmoe.so (C ABI in include/moe.h); `inputs`
draws the seeded synthetic workloads; `build` compiles the library for sm_100a.
"""
from . import inputs  # noqa: F401

__all__ = ["inputs", "moe", "build"]
