"""fp64 CPU oracle (test infrastructure only; see ``oracle.attention``).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The CUDA library never does.
"""
from .attention import (  # noqa: F401
    attn_scores_ref,
    attn_probs_ref,
    attn_fwd_ref,
    attn_fwd_rows_ref,
    attn_bwd_ref,
    online_fwd_ref,
    fa1_fwd_ref,
    gqa_fwd_ref,
    gqa_bwd_ref,
    blocksparse_fwd_ref,
    blocksparse_bwd_ref,
    merge_partials_ref,
    attn_bwd_partial_ref,
    attn_dq_rows_ref,
    ring_fwd_ref,
    ring_bwd_ref,
)
from .fp8 import (  # noqa: F401
    E4M3_MAX,
    e4m3_round_ref,
    hadamard_ref,
    rotate_ref,
    quantize_rows_ref,
    quantize_cols_ref,
    fp8_inputs_ref,
    fp8_attn_fwd_ref,
)
