"""spatial_spectral_attention_b200: the spatial-spectral coupling of deep
functional maps (dense and Geo-FlashAttention) as sm_100a CUDA kernels behind
the C ABI of include/ssc.h.  `api` is the Python binding of that ABI."""
from . import synth  # noqa: F401  (seeded input generator)

__all__ = ["api", "synth", "build"]
