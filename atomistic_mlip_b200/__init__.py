"""B200-native on-the-fly SO(2) equivariant attention (E2Former-V2 hot path).

Importing the package loads nothing native; the CUDA library is loaded on
first use by :mod:`atomistic_mlip_b200.e2f`, which raises if it is missing.
"""
__all__ = ["e2f", "workloads"]
