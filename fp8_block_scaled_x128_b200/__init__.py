"""Fine-grained-scaled FP8 GEMM for B200 (sm_100a).

The entry points live in the CUDA library libfp8gemm.so (C ABI:
include/fp8gemm.h).  Their Python bindings are loaded on first use, so that
importing this package (for example for the input generator in `synth`) does
not need the library; calling a GEMM without it raises ImportError.
"""
from __future__ import annotations

import importlib

__all__ = ["fp8_gemm_nt", "m_grouped_fp8_gemm_nt_contiguous", "m_grouped_fp8_gemm_nt_masked"]


def __getattr__(name):
    if name in __all__:
        return getattr(importlib.import_module(__name__ + ".gemm"), name)
    raise AttributeError(name)
