"""Exact tiled attention for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libfa_sm100.so`` (include/fa.h); the
module :mod:`exact_tiled_attention_40_b200.fa` is its Python binding.  Importing
this package loads nothing; the library is loaded on first use.  Also here:
:mod:`ring` (sequence-sharded forward over ranks), :mod:`sharding` (batch, head
group and ragged-batch partitions), :mod:`inputs` (seeded synthetic inputs),
:mod:`run_case` (time one workload) and :mod:`build` (compile the library).
"""

__all__ = ["fa", "inputs", "ring", "sharding", "run_case", "build"]
