"""B200-native (sm_100a) Infini-attention forward pass.

The compute path is the C-ABI CUDA library ``libinfini_attn.so`` built from ``csrc/``;
``binding`` marshals torch tensors into it.  ``workloads`` holds the seeded synthetic
inputs.  Importing the package does not load the CUDA library; ``binding`` does, and it
raises if the library is missing.
"""
__all__ = ["binding", "workloads"]
