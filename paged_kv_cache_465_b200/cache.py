"""PagedKVCache: one layer's block pool on the GPU plus its host block allocator.

A convenience object over the C ABI: the pool tensors (K, V and, for fp8 / int8, the
per-(block, kv head) scales and int8 zero points) live in torch-allocated device memory,
the allocator is the library's native one (with automatic prefix caching), and every
device operation (write, copy, decode, prefill) is one of the library's kernels.
"""
from __future__ import annotations

from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

from . import (BlockAllocator, copy_blocks, paged_attn_decode, paged_attn_prefill,
               reshape_and_cache, workspace_size, decode_desc_for)

_TORCH_DTYPE = {"f32": "float32", "bf16": "bfloat16", "fp8": "uint8", "int8": "int8"}


class PagedKVCache:
    def __init__(self, num_blocks: int, num_kv_heads: int, head_dim: int, kv_dtype: str,
                 block_size: int = 16, device="cuda", order: Optional[Sequence[int]] = None):
        import torch
        self.torch = torch
        self.num_blocks, self.num_kv_heads, self.head_dim = num_blocks, num_kv_heads, head_dim
        self.block_size, self.kv_dtype = block_size, kv_dtype
        dt = getattr(torch, _TORCH_DTYPE[kv_dtype])
        shape = (num_blocks, num_kv_heads, block_size, head_dim)
        self.k_cache = torch.zeros(shape, dtype=dt, device=device)
        self.v_cache = torch.zeros(shape, dtype=dt, device=device)
        if kv_dtype in ("fp8", "int8"):
            self.k_scales = torch.ones((num_blocks, num_kv_heads), dtype=torch.float32, device=device)
            self.v_scales = torch.ones((num_blocks, num_kv_heads), dtype=torch.float32, device=device)
        else:
            self.k_scales = self.v_scales = None
        if kv_dtype == "int8":
            self.k_zeros = torch.zeros((num_blocks, num_kv_heads), dtype=torch.int32, device=device)
            self.v_zeros = torch.zeros((num_blocks, num_kv_heads), dtype=torch.int32, device=device)
        else:
            self.k_zeros = self.v_zeros = None
        self.alloc = BlockAllocator(num_blocks, block_size, order)

    # ---- host bookkeeping ----------------------------------------------------------------
    def add_seq(self, seq: int, num_tokens: int) -> np.ndarray:
        return self.alloc.add_seq(seq, num_tokens)

    def fork(self, parent: int, child: int) -> None:
        self.alloc.fork(parent, child)

    def append(self, seq: int, num_tokens: int) -> Tuple[np.ndarray, List[Tuple[int, int]]]:
        return self.alloc.append(seq, num_tokens)

    def append_batch(self, seqs, num_tokens=1) -> Tuple[np.ndarray, np.ndarray]:
        """A decode step's bookkeeping in one library call (all or nothing): the new tokens'
        slots, sequence after sequence, and the copy-on-write pairs to copy first."""
        return self.alloc.append_batch(seqs, num_tokens)

    def free_seq(self, seq: int) -> None:
        self.alloc.free_seq(seq)

    def block_tables(self, seqs: Sequence[int], max_blocks: int):
        return self.torch.from_numpy(self.alloc.padded_tables(seqs, max_blocks))

    # ---- device operations -------------------------------------------------------------
    def write(self, k, v, slots, stream=None) -> None:
        reshape_and_cache(k, v, self.k_cache, self.v_cache, slots, k_scales=self.k_scales,
                          v_scales=self.v_scales, k_zeros=self.k_zeros, v_zeros=self.v_zeros,
                          stream=stream)

    def copy(self, pairs, stream=None) -> None:
        if pairs is not None and pairs.shape[0] > 0:
            copy_blocks(self.k_cache, self.v_cache, pairs, k_scales=self.k_scales,
                        v_scales=self.v_scales, k_zeros=self.k_zeros, v_zeros=self.v_zeros,
                        stream=stream)

    def workspace_bytes(self, q, block_tables, max_context_len: int, partition_size: int) -> int:
        return workspace_size(decode_desc_for(q, self.k_cache, block_tables, partition_size),
                              max_context_len)

    def decode(self, q, block_tables, context_lens, scale: float, out, *, max_context_len: int,
               partition_size: int = 0, lse_out=None, workspace=None, stream=None):
        return paged_attn_decode(q, self.k_cache, self.v_cache, block_tables, context_lens,
                                 scale, out, max_context_len=max_context_len,
                                 partition_size=partition_size, k_scales=self.k_scales,
                                 v_scales=self.v_scales, k_zeros=self.k_zeros,
                                 v_zeros=self.v_zeros, lse_out=lse_out, workspace=workspace,
                                 stream=stream)

    def prefill(self, q, block_tables, context_lens, query_start, scale: float, out, *,
                max_query_len: int, max_context_len: int, lse_out=None, stream=None):
        return paged_attn_prefill(q, self.k_cache, self.v_cache, block_tables, context_lens,
                                  query_start, scale, out, max_query_len=max_query_len,
                                  max_context_len=max_context_len, k_scales=self.k_scales,
                                  v_scales=self.v_scales, k_zeros=self.k_zeros,
                                  v_zeros=self.v_zeros, lse_out=lse_out, stream=stream)
