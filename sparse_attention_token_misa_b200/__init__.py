"""B200-native (sm_100a) MISA / MISA-dagger / HISA token indexer, and the
sparse attention over the tokens it selects.

The compute path is libmisa.so (C ABI in include/misa.h, CUDA kernels under
csrc/); this package is its Python binding: the same entry points taking torch
device tensors (`_native`), and the four indexers as preallocated call
sequences (`indexer`).
"""
from . import _native
from ._native import (MisaError, alloc_workspace, append_keys, block_stats, error_query, error_reset,  # noqa: F401
                      gather_candidates, hier_rerank, hisa_block_filter, index_decode, index_score, index_score_blocks, lib, num_windows,
                      route_heads,
                      shard_prefix, sparse_mla, topk, workspace_bytes)
from .indexer import DenseIndexer, HisaIndexer, MisaDaggerIndexer, MisaIndexer  # noqa: F401
from .sharded import ShardedMisaIndexer, TorchShardComm, shard_bounds  # noqa: F401

__all__ = [
    "MisaError", "alloc_workspace", "append_keys", "block_stats", "error_query", "error_reset",
    "gather_candidates", "hier_rerank", "shard_prefix", "ShardedMisaIndexer", "TorchShardComm", "shard_bounds",
    "hisa_block_filter", "index_decode", "index_score", "index_score_blocks", "lib", "num_windows", "route_heads", "sparse_mla", "topk", "workspace_bytes",
    "DenseIndexer", "HisaIndexer", "MisaDaggerIndexer", "MisaIndexer",
]
