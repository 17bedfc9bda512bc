"""CPU oracle for indexer-routed token-sparse attention with a shared index.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously
correct definition that the CUDA library is checked against.  Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import or call it; the product path (the ``libsa.so``
C ABI and its Python binding) never does, and shares no code with it.

Everything is numpy in float64.  Library primitives (matmul, sort, exp) are
used as single steps; there is no blocking, fusion or reordering beyond the
definitions the functions cite.  Pins that tie each function to facts other
than itself live in ``tests/test_oracle_pins.py``.
"""
from .reference import (  # noqa: F401
    bf16_bits_to_f64,
    e4m3_bits_to_f64,
    n_candidates,
    index_scores,
    index_scores_multihead,
    topk_select,
    index_topk,
    attention_over_rows,
    sparse_attention,
    sparse_attention_decode,
    gist_route_unfold,
    hier_gist_route_unfold,
    layer_owners,
    index_overlap,
    greedy_pattern,
    kv_cache_gib,
    pair_counts,
)
