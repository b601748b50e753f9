"""B200-native paged decode attention and paged cache write.

The compute path is the C-ABI library ``libpaged_attn.so`` (hand-written
sm_100a CUDA); ``binding`` marshals torch tensors into its calls.  Importing
this package does not load the library; the first ``PagedAttention(...)``
does, and raises if it is missing (there is no CPU fallback).
"""

__all__ = ["binding", "workloads"]
