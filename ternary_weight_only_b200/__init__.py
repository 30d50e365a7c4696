"""Ternary-g128 weight-only matmul for NVIDIA B200 (sm_100a).

``ternary_weight_only_b200.tern`` is the binding of the C library libtern.so
(include/tern.h); ``ternary_weight_only_b200.synth`` draws seeded synthetic
inputs; ``ternary_weight_only_b200.build`` compiles the library with nvcc.
"""
__all__ = ["tern", "synth", "build"]
