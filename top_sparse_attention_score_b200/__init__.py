"""QSA sparse-attention step on NVIDIA B200 (sm_100a).

The computation lives in the CUDA library ``libqsa_b200.so`` (C ABI:
include/qsa.h); ``qsa`` is its ctypes binding.  Build the library with
``top_sparse_attention_score_b200.build.build()``.
"""
from . import qsa  # noqa: F401

__all__ = ["qsa"]
