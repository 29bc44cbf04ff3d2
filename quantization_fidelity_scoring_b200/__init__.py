"""B200-native teacher-forced KL(reference || candidate) scoring.

The compute lives in libkld.so (hand-written sm_100a kernels behind the C ABI
of include/kld.h); this package is its Python binding.
"""
from . import _lib
from .api import (KldError, kld_from_hidden_shared_head, kld_full_vocab, kld_full_vocab_workspace_size,
                  kld_paired_compare, kld_paired_workspace_size, kld_reduce_shard_block_bytes,
                  kld_reduce_shard_step, kld_reduce_shard_workspace_size, kld_reduce_stats,
                  kld_reduce_workspace_size, kld_shared_head_workspace_size, kld_sparse_capture,
                  kld_sparse_capture_workspace_size, kld_sparse_ref_score, kld_sparse_ref_workspace_size,
                  kld_topk_tail, paired_from_device, stats_from_device, stats_to_dict)

__all__ = ["KldError", "kld_from_hidden_shared_head", "kld_shared_head_workspace_size", "kld_full_vocab",
           "kld_full_vocab_workspace_size", "kld_topk_tail", "kld_reduce_stats", "kld_reduce_workspace_size",
           "kld_sparse_ref_score", "kld_sparse_ref_workspace_size", "kld_sparse_capture",
           "kld_sparse_capture_workspace_size", "kld_reduce_shard_step", "kld_reduce_shard_block_bytes",
           "kld_reduce_shard_workspace_size", "kld_paired_compare", "kld_paired_workspace_size",
           "paired_from_device", "stats_from_device", "stats_to_dict", "load_library"]


def load_library():
    """Load libkld.so (raises ImportError when it has not been built)."""
    return _lib.load()
