"""combine_overlap_b200: one Mixture-of-Experts layer on a B200 (sm_100a), with
the gate-weighted combine overlapped with the expert GEMM at tile granularity.

The compute path is the C-ABI library ``libmoe_b200.so`` (CUDA, built from
``csrc/``); ``combine_overlap_b200.moe`` is a thin ctypes binding over it.
Importing the package itself loads nothing, so the seeded input generator
(``combine_overlap_b200.synth``) is usable without a GPU.
"""
__all__ = ["synth", "moe"]
