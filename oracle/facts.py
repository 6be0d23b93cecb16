"""Closed-form sizes and ratios printed on the pages (test infrastructure only).

Each function states one formula from the pages; the CPU tests pin it against the numbers
the pages print for their worked examples (``tests/golden/*.json``).
"""
from __future__ import annotations

import math


def kv_cache_bytes(num_layers: int, num_kv_heads: int, head_dim: int, dtype_bytes: int,
                   tokens: int, batch: int = 1) -> int:
    """KV bytes = num_layers * 2 (K and V) * batch * num_kv_heads * seq_len * head_dim * bytes.

    [KVPaged] "Why does the KV cache eat memory" (the byte formula) and [KVFail] Key Points
    (capacity estimate: 2 x layers x KV heads x head dim x bytes x active tokens).
    """
    return num_layers * 2 * batch * num_kv_heads * tokens * head_dim * dtype_bytes


def blocks_for_tokens(tokens: int, block_size: int = 16) -> int:
    """Allocated blocks B_r = ceil(T_r / B_s): [Ch4PA] Theorem 1, proof."""
    return -(-tokens // block_size)


def last_block_fill(tokens: int, block_size: int = 16) -> int:
    """Tokens held by the last block: [KVPaged] block-table example (40 tokens -> 16+16+8)."""
    if tokens == 0:
        return 0
    return tokens - block_size * (blocks_for_tokens(tokens, block_size) - 1)


def paged_waste_fraction(lengths, block_size: int = 16) -> float:
    """Unused slots / allocated slots over a batch (internal fragmentation of the last
    blocks): the quantity bounded by [Ch4PA] Theorem 1 (waste <= B_s / T)."""
    alloc = sum(blocks_for_tokens(t, block_size) * block_size for t in lengths)
    used = sum(lengths)
    return (alloc - used) / alloc if alloc else 0.0


def waste_bound(min_len: int, block_size: int = 16) -> float:
    """[Ch4PA] Theorem 1: waste <= B_s / T for a batch whose lengths are all >= T."""
    return block_size / min_len


def internal_fragmentation_contiguous(tokens: int, max_tokens: int) -> float:
    """Naive contiguous reservation: IFrag = 1 - T / T_max ([Ch4PA], "three defects")."""
    return 1.0 - tokens / max_tokens


def sharing_savings_prefix_only(num_requests: int) -> float:
    """R requests sharing one prefix keep one copy: savings = 1 - 1/R ([Ch4PA], OS paging
    section, copy-on-write paragraph)."""
    return 1.0 - 1.0 / num_requests


def sharing_savings(num_requests: int, prefix: int, suffix: float) -> float:
    """Savings = (R-1) p / (R (p + s)) ([Ch4PA], "Prefix Caching")."""
    R = num_requests
    return (R - 1) * prefix / (R * (prefix + suffix))


def block_table_bytes(num_requests: int, max_tokens: int, block_size: int = 16,
                      entry_bytes: int = 4) -> int:
    """Block-table memory: one int32 entry per logical block of the longest allowed context
    per request ([Ch4PA], "vLLM 4-layer architecture", KV Cache Manager paragraph)."""
    return num_requests * math.ceil(max_tokens / block_size) * entry_bytes
