"""B200-native variable-length (packed, cu_seqlens-indexed) attention forward.

The compute path is the C-ABI library ``libvarlen_attn.so`` built from
``csrc/`` for sm_100a; ``binding`` marshals torch tensors into its calls.
Importing this package loads nothing; ``binding.load()`` does, and raises if
the library is missing.
"""
__all__ = ["binding", "workloads"]
