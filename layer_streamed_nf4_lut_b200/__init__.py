"""Layer-streamed NF4 + LoRA training step for one B200 (sm_100a).

The compute lives in libsoup.so (CUDA kernels + C-ABI, include/soup.h); this package is its
Python binding.  `from layer_streamed_nf4_lut_b200 import model` loads the library and raises
if it has not been built.
"""
__all__ = ["model", "build"]
