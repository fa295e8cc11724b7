"""MoE token dispatch and combine for one B200 (sm_100a).

The compute lives in the CUDA library ``libmoe_dispatch.so`` built from
``csrc/``; ``ops`` holds a thin ctypes binding with the C entry points' names.
Importing this package does not load the library; the first call does, and
fails loudly if it is missing.
"""
__all__ = ["workloads"]
