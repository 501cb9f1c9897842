"""CPU oracle for KVzip scoring, global selection and KV compaction.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The library
(``attention_score_reduction_b200``) never imports it and never falls back to
it: the CUDA path and this oracle share no code.

See ``oracle.kvzip_oracle`` for the definitions and the passages they follow.
"""
from .kvzip_oracle import (  # noqa: F401
    causal_self_mask,
    chunk_logits,
    softmax_rows,
    unit_chunk_scores,
    score_chunk,
    score_context,
    keep_count,
    select,
    compact,
    head_scores,
    decode_attention,
    unit_chunk_colsums,
    score_chunk_sum,
    token_scores,
    select_per_head,
    expand_keep,
)
