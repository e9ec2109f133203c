"""SLAY spherical Yat-kernel linear attention on B200 (sm_100a).

The compute path is the C-ABI library libslay.so (CUDA kernels for sm_100a);
`binding` marshals torch tensors into its entry points.  `workloads` holds the
seeded synthetic input recipe.  Importing the package does not load the library;
the first call through `binding` does, and fails loudly if it is missing.
"""
__all__ = ["binding", "workloads"]
