"""Pins of the oracle's automatic prefix caching (chained block hashes, reuse, eviction).

Against: SHA-256 known answers built from explicitly spelled-out bytes (hashlib over
little-endian int32 tokens, the parent digest first); the prefix property (a block's hash
names the whole prefix up to it, so a change in block i changes the hashes of blocks >= i
and no earlier one); the pages' sharing-savings formula for a common system prompt; a
hand-worked least-recently-used eviction trace; atomic failure.
"""
import hashlib

import numpy as np
import pytest

from oracle import facts
from oracle.paged import NoBlocks, RefAllocator


def _le_bytes(tokens):
    return b"".join(int(t).to_bytes(4, "little", signed=True) for t in tokens)


def _hashes(a, tokens):
    """The chained hashes of the full blocks of ``tokens``, via the oracle."""
    B = a.block_size
    out = []
    for i in range(len(tokens) // B):
        out.append(a.chain_hash(out[-1] if out else None, tokens[i * B:(i + 1) * B]))
    return out


def test_known_answers():
    a = RefAllocator(4, 16)
    blk0 = list(range(16))
    blk1 = [-1, 2 ** 31 - 1, -2 ** 31] + list(range(1000, 1013))
    h0 = hashlib.sha256(_le_bytes(blk0)).digest()
    h1 = hashlib.sha256(h0 + _le_bytes(blk1)).digest()
    assert _hashes(a, blk0 + blk1 + [5, 6]) == [h0, h1]
    # the bytes of the first token are 00 00 00 00, of the second 01 00 00 00
    assert _le_bytes([1])[:1] == b"\x01"


def test_prefix_property():
    rng = np.random.default_rng(3)
    a = RefAllocator(4, 8)
    base = rng.integers(0, 50000, 8 * 6).tolist()
    hb = _hashes(a, base)
    assert len(set(hb)) == 6
    for i in range(6):
        alt = list(base)
        alt[8 * i + int(rng.integers(0, 8))] += 1
        ha = _hashes(a, alt)
        assert ha[:i] == hb[:i]
        assert all(x != y for x, y in zip(ha[i:], hb[i:]))
    # equal block contents at different depths hash differently (the prefix is named)
    rep = list(range(8)) * 3
    hr = _hashes(a, rep)
    assert len(set(hr)) == 3


def test_hits_are_a_leading_run_of_full_blocks():
    B = 16
    a = RefAllocator(16, B)
    x = list(range(3 * B + 5))                   # 3 full blocks + 5 tokens
    _, c = a.add_seq_tokens(0, x)
    assert c == 0 and len(a.cache) == 3          # the partial last block is not registered
    y = list(x[:3 * B]) + [9] * 7
    _, c = a.add_seq_tokens(1, y)
    assert c == 3 * B and a.block_table(1)[:3] == a.block_table(0)[:3]
    z = [777] + x[1:]                            # block 0 differs: no later block can hit
    _, c = a.add_seq_tokens(2, z)
    assert c == 0 and set(a.block_table(2)).isdisjoint(a.block_table(0))
    w = x[:B] + [0] * B + x[2 * B:3 * B]         # block 1 differs: only block 0 hits
    _, c = a.add_seq_tokens(3, w)
    assert c == B
    for b in a.block_table(0)[:3]:
        assert a.ref_count(b) == (3 if b == a.block_table(0)[0] else 2)


def test_shared_system_prompt_savings():
    """R requests with a common p-token prompt and s private tokens each: the reused share of
    all tokens is the pages' (R-1) p / (R (p + s)) for the block-aligned part of the prompt."""
    R, p, sfx, B = 100, 200, 50, 16
    rng = np.random.default_rng(2)
    prompt = rng.integers(0, 32000, p).tolist()
    a = RefAllocator(512, B)
    cached = [a.add_seq_tokens(r, prompt + rng.integers(0, 32000, sfx).tolist())[1]
              for r in range(R)]
    assert cached[0] == 0 and all(c == (p // B) * B for c in cached[1:])
    assert 512 - a.num_free() == 16 + (R - 1) * (16 - 12)
    assert sum(cached) / (R * (p + sfx)) == pytest.approx(
        facts.sharing_savings(R, 192, p + sfx - 192))
    assert (a.hit_blocks, a.evictions) == ((R - 1) * 12, 0)


def test_lru_eviction_trace():
    """Worked by hand from the policy: freed blocks queue at the back with their hashes; a
    hit takes a waiting block out of the queue; popping a waiting block evicts its hash."""
    B = 16
    a = RefAllocator(8, B)
    x = list(range(1, 33))
    y = list(range(100, 132))
    a.add_seq_tokens(0, x)                       # blocks 0, 1
    a.add_seq_tokens(1, y)                       # blocks 2, 3
    a.free_seq(0)
    a.free_seq(1)
    assert list(a.free) == [4, 5, 6, 7, 0, 1, 2, 3] and len(a.cache) == 4
    a.add_seq(2, 4 * B)                          # 4..7
    a.add_seq(3, 2 * B)                          # 0, 1: x's entries evicted
    assert a.block_table(3) == [0, 1] and a.evictions == 2 and len(a.cache) == 2
    a.free_seq(2)
    assert list(a.free) == [2, 3, 4, 5, 6, 7]
    _, c = a.add_seq_tokens(5, y + [7])
    assert c == 32 and a.block_table(5) == [2, 3, 4]
    _, c = a.add_seq_tokens(4, x)
    assert c == 0 and a.block_table(4) == [5, 6]
    assert a.hit_blocks == 2


def test_shortage_with_hits_changes_nothing():
    a = RefAllocator(4, 16)
    p = list(range(48))
    a.add_seq_tokens(0, p)
    a.free_seq(0)
    a.add_seq(1, 16)                             # takes block 3; blocks 0..2 wait, cached
    before = (list(a.free), dict(a.cache), list(a.refs), a.hit_blocks, a.evictions)
    with pytest.raises(NoBlocks):
        a.add_seq_tokens(2, p + list(range(100, 140)))
    assert (list(a.free), dict(a.cache), list(a.refs), a.hit_blocks, a.evictions) == before
    _, c = a.add_seq_tokens(3, p)
    assert c == 48 and a.num_free() == 0
