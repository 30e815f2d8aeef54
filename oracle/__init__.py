"""fp64 CPU oracle of the Sparse-to-Dense hot path.

TEST INFRASTRUCTURE: imported only by the test-suite, ``__graft_entry__.smoke()``
and the CPU-baseline legs of ``bench.py``; never by the library.
"""
from .std_oracle import (  # noqa: F401
    accept_prefix,
    attend,
    attend_partial,
    attn_range_partial,
    decode_round,
    dense_verify_attn,
    gather_sparse,
    kv_append,
    kv_commit,
    merge_candidates,
    merge_partials,
    merge_rowstats,
    select_topk,
    selection_scores,
    selection_rowstats,
    selection_scores_causal,
    selection_scores_given_rowstats,
    softmax,
    sparse_decode_attn,
    streaming_indices,
    topk_candidates,
    topk_indices,
)
