"""Block-sparse causal prefill attention (FlashPrefill style) for B200 / sm_100a.

The compute path is a C-ABI shared library of hand-written CUDA kernels
(``libflashprefill.so``, built in-tree); ``binding`` is its thin ctypes wrapper
and ``workloads`` the seeded synthetic input generator.
"""
__all__ = ["binding", "workloads"]
