"""Exact tiled attention for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libfa_sm100.so`` (include/fa.h); the
module :mod:`exact_tiled_attention_40_b200.fa` is its Python binding.  Importing
this package loads nothing; the library is loaded on first use.
"""

__all__ = ["fa", "inputs"]
