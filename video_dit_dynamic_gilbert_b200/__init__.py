"""B200-native Adaptive Block-Sparse Attention (ASA / ASA_G) for video DiTs.

The compute path lives in libasa.so (CUDA for sm_100a, C ABI in include/asa.h);
`video_dit_dynamic_gilbert_b200.asa` is its Python binding.
"""
__all__ = ["asa"]
