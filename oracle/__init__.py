"""fp64 CPU oracle of the top-k routed MoE SwiGLU layer forward.

TEST INFRASTRUCTURE: imported only by the tests, the smoke check and the
benchmark's CPU-baseline leg; never by the product path.
"""
