"""Ulysses sequence parallelism on one B200: the attention layer with P
logical ranks held in one GPU's HBM.

The compute path is the C-ABI library ``libulysses.so`` (hand-written sm_100a
CUDA kernels); :mod:`long_context_sequence_all_b200.ulysses` is its thin
ctypes binding.  Importing this package loads nothing; the library is loaded
on first use and a missing or unloadable library is a hard error.
"""
__all__ = ["ulysses", "workloads"]
