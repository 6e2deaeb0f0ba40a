"""B200-native differential-attention forward pass (prefill, grouped prefill,
single-query decode) behind the C-ABI library ``libdiffattn``.

The CUDA library is loaded on first use by :mod:`.ops`; importing the package
itself loads nothing, so the input generators work on machines without a GPU.
"""
__all__ = ["inputs", "ops"]
