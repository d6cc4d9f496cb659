"""fp64 CPU oracle for exact tiled attention (test infrastructure only).

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of bench.py may
import this package.  The library never does.
"""
from .attention_fp64 import (  # noqa: F401
    attention,
    attention_backward,
    attention_rows,
    blockwise_attention,
    causal_allowed,
    decode_paged,
    gather_paged_kv,
    kv_head_of,
    merge_partials,
    paged_prefill,
    softmax_rows,
    varlen_attention,
)
