"""libintfa: INT8-quantised attention forward pass (INT-FlashAttention style)
on B200 (sm_100a).

The compute lives in ``csrc/`` (CUDA kernels behind a C ABI, built into
``libintfa.so``); ``intfa`` is the thin ctypes binding and ``workloads`` the
seeded input generator.
"""
__all__ = ["intfa", "workloads"]
