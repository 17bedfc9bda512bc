"""B200-native indexer-routed token-sparse attention with a cross-layer shared index.

The product is the C ABI ``libsa.so`` (declared in ``include/sa.h``, sources
in ``csrc/``).  ``shared_top_routing_b200.sa`` is its Python binding; it only
marshals arguments.  Build with ``python -m shared_top_routing_b200.build``.
"""
from .sa import (  # noqa: F401
    SA_ERR_CUDA,
    SA_ERR_INVALID_ARG,
    SA_ERR_STALE_INDEX,
    SA_ERR_UNSUPPORTED,
    SA_ERR_WORKSPACE,
    SA_OK,
    IndexCache,
    SAError,
    lib,
    sa_gather_rows,
    sa_gist_route_unfold,
    sa_hier_gist_route_unfold,
    sa_index_overlap,
    sa_index_pattern_greedy,
    sa_index_score_topk,
    sa_index_score_topk_mh,
    sa_index_score_topk_fp8,
    sa_workspace_status,
    sa_sparse_attn_decode,
    sa_sparse_attn_decode_rows,
    sa_sparse_attn_prefill,
)

__all__ = [
    "SA_ERR_CUDA",
    "SA_ERR_INVALID_ARG",
    "SA_ERR_STALE_INDEX",
    "SA_ERR_UNSUPPORTED",
    "SA_ERR_WORKSPACE",
    "SA_OK",
    "IndexCache",
    "SAError",
    "lib",
    "sa_gather_rows",
    "sa_gist_route_unfold",
    "sa_hier_gist_route_unfold",
    "sa_index_overlap",
    "sa_index_pattern_greedy",
    "sa_index_score_topk",
    "sa_index_score_topk_mh",
    "sa_index_score_topk_fp8",
    "sa_workspace_status",
    "sa_sparse_attn_decode",
    "sa_sparse_attn_decode_rows",
    "sa_sparse_attn_prefill",
]
