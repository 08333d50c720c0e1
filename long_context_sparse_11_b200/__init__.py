"""B200 (sm_100a) DeepSeek-Sparse-Attention step with IndexShare.

The CUDA library ``libdsa.so`` (C ABI: include/dsa.h) holds every kernel of the path;
this package is its Python binding.  Build it with ``long_context_sparse_11_b200.build``.
"""
from .binding import (  # noqa: F401
    CacheView, IndexHandle, GroupArgs, DsaError, IndexShareGroup, load, dense_view, paged_view,
    quant_e4m3, cache_write_e4m3, indexer_score, topk, topk_no_alloc, sparse_mla_attn, sync_status,
    layer_is_full, layer_producer, indexer_project, mla_latent, rope_query, ROPE_THETA,
    split_candidates, split_merge, combine_partials, CacheWriteBatch,
    DSA_BF16, DSA_E4M3, EXPORTS,
)
