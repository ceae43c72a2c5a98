"""B200-native (sm_100a) paged decode attention: the cache write and the
decode-step attention over a block-table-addressed KV cache.

The compute lives in ``libpa.so`` (CUDA kernels behind the C ABI of
``include/pa.h``); this package only marshals torch tensors into those calls.

    from paged_kv_cache_444_b200 import pa_reshape_and_cache, pa_decode
"""
from __future__ import annotations

import torch

from ._lib import (DecodePlan, HostStep, PagedAttentionError, load, pa_check_error, pa_copy_blocks, pa_decode,
                   pa_decode_fp8, pa_decode_noalloc, pa_decode_shared_prefix, pa_decode_split,
                   pa_decode_split_fp8, pa_prefill, pa_reduce, pa_reshape_and_cache,
                   pa_reshape_and_cache_fp8, pa_selftest_wait_timeout)

__all__ = [
    "PagedAttentionError", "load", "pa_reshape_and_cache", "pa_decode", "pa_decode_split",
    "pa_reduce", "pa_check_error", "pa_decode_noalloc", "pa_decode_shared_prefix",
    "pa_copy_blocks", "pa_reshape_and_cache_fp8", "pa_decode_fp8", "pa_decode_split_fp8",
    "pa_prefill", "pa_selftest_wait_timeout", "SplitWorkspace", "decode_step", "HostStep",
    "DecodePlan",
]


class SplitWorkspace:
    """Caller-owned fp32 scratch for pa_decode_split / pa_reduce
    (tmp_out [S, H, P, D], max_logits and exp_sums [S, H, P])."""

    def __init__(self, num_seqs: int, num_heads: int, head_dim: int, max_partitions: int,
                 device: torch.device | str):
        shape = (num_seqs, num_heads, max_partitions)
        self.tmp_out = torch.empty(shape + (head_dim,), dtype=torch.float32, device=device)
        self.max_logits = torch.empty(shape, dtype=torch.float32, device=device)
        self.exp_sums = torch.empty(shape, dtype=torch.float32, device=device)

    @property
    def max_partitions(self) -> int:
        return self.max_logits.shape[-1]


def decode_step(query, key, value, key_cache, value_cache, slot_mapping, block_tables,
                context_lens, scale: float, out: torch.Tensor | None = None,
                partition_size: int = 0, workspace: SplitWorkspace | None = None,
                stream=None) -> torch.Tensor:
    """One decode step of one attention layer: write this step's K/V rows
    (pa_reshape_and_cache), then attend (pa_decode, or pa_decode_split +
    pa_reduce when partition_size > 0).  All tensors live on one CUDA device."""
    if out is None:
        out = torch.empty_like(query)
    if key is not None and key.shape[0] > 0:
        pa_reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, stream)
    if partition_size > 0:
        if workspace is None:
            bs = key_cache.shape[1]
            P = (block_tables.shape[1] * bs + partition_size - 1) // partition_size
            workspace = SplitWorkspace(query.shape[0], query.shape[1], query.shape[2], P,
                                       query.device)
        pa_decode_split(workspace.tmp_out, workspace.max_logits, workspace.exp_sums, query,
                        key_cache, value_cache, block_tables, context_lens, scale,
                        partition_size, stream)
        pa_reduce(out, workspace.tmp_out, workspace.max_logits, workspace.exp_sums,
                  context_lens, partition_size, stream)
    else:
        pa_decode(out, query, key_cache, value_cache, block_tables, context_lens, scale, stream)
    return out
