"""libserq: B200-native SERQ quantized linear (sm_100a).

The CUDA path is reached through :mod:`w4a4_rank_gemm_b200.serq`, which loads
the in-tree ``libserq.so`` and raises if it is missing.  This package module
itself imports nothing heavy so that the seeded input generators in
:mod:`w4a4_rank_gemm_b200.synth` can be used without a GPU.
"""
__all__ = ["serq", "synth"]
