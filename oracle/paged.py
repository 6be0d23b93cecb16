"""Paged KV-cache bookkeeping and cache writes of the oracle (test infrastructure only).

Cache layout (a reading: the pages give no memory layout): ``cache[num_blocks][num_kv_heads]
[block_size][head_dim]``, i.e. every (physical block, kv head) tile is contiguous. The oracle
stores the cache in its storage codes: float32 values, uint16 bf16 bits or uint8 E4M3 codes.

[KVPaged] "PagedAttention: OS virtual-memory style management": the cache is cut into small
fixed-size blocks, one block is allocated as tokens accumulate, and a per-request block
table maps logical token positions to physical blocks (16-token example: 40 tokens ->
[blk0, blk3, blk5], 20 tokens -> [blk1, blk2]).
[Ch4PA] "PagedAttention algorithm": logical block id -> physical block address, physical
addresses need not be contiguous; "OS paging": a free list of fixed-size units always
serves an allocation while enough units remain.
[KVFail] Key Points: when free blocks are short the allocation fails (read: the call fails
and changes nothing); blocks are handed out from a free queue.
[KVPaged] "Prefix sharing and copy-on-write" and [Ch4PA] "Prefix Caching": sequences with a
common prefix point at the same physical blocks, a ref_count tracks the sharers, and a
shared block is copied only when a writer modifies it.
"""
from __future__ import annotations

import copy
import hashlib
from collections import deque
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

from .codecs import bf16_encode, bf16_decode, e4m3_encode, int8_encode


class NoBlocks(Exception):
    """The free queue holds fewer blocks than the call needs; nothing was changed."""


class InvalidCall(Exception):
    """Unknown / duplicate sequence id or a bad argument; nothing was changed."""


def slot_of(block_table_row: Sequence[int], pos: int, block_size: int) -> int:
    """Slot of logical token ``pos``: physical block * block_size + offset in the block."""
    return int(block_table_row[pos // block_size]) * block_size + pos % block_size


class RefAllocator:
    """Reference block allocator.

    Policy (readings, stated once):
    * the free queue is FIFO, initialised with ``order`` (default 0..N-1); allocation pops
      from the front; a block whose ref_count drops to 0 is pushed to the back;
    * ``add_seq(s, n)`` allocates ceil(n/B) blocks in logical order;
    * ``fork(p, c)`` gives ``c`` a copy of ``p``'s block table and length and increments the
      ref_count of every block in it;
    * ``append(s, n)``: if the last block is partially filled AND shared (ref_count > 1) it is
      copied first: one new block is popped, the pair (old, new) is reported, ``old`` loses a
      reference and ``new`` takes its place in the table; then one block is popped for every
      new 16-token boundary crossed. A full shared block is never written, so it is never
      copied. At most one copy pair per call;
    * every call checks first and changes nothing when it fails.

    Automatic prefix caching ([Ch4PA] "Prefix Caching": a SHA-256 hash of the prefix
    identifies identical blocks, hits raise ref_count; [KVPaged] "Prefix cache lifetime and
    invalidation": hits skip recomputation, eviction is least recently used; [KVFail] Key
    Points: a cached block is evicted when the free queue hands it out again):
    * full block i of a sequence added with ``add_seq_tokens`` has the chained hash
      h_i = sha256(h_{i-1} + little-endian int32 tokens of block i), h_{-1} = b"";
    * the longest run of leading full blocks with cached hashes is reused (a waiting block
      is taken out of the free queue), the other blocks are popped, the new full blocks
      registered;
    * a freed block keeps its entry while it waits in the free queue; popping it evicts it.
    """

    def __init__(self, num_blocks: int, block_size: int = 16,
                 order: Optional[Sequence[int]] = None):
        if num_blocks <= 0 or block_size <= 0:
            raise InvalidCall("sizes")
        self.num_blocks = num_blocks
        self.block_size = block_size
        if order is None:
            order = range(num_blocks)
        order = [int(b) for b in order]
        if sorted(order) != list(range(num_blocks)):
            raise InvalidCall("order must be a permutation of the block ids")
        self.free: deque = deque(order)
        self.refs: List[int] = [0] * num_blocks
        self.tables: Dict[int, List[int]] = {}
        self.lens: Dict[int, int] = {}
        self.cache: Dict[bytes, int] = {}        # chained hash -> block
        self.block_hash: Dict[int, bytes] = {}   # block -> its hash
        self.hit_blocks = 0
        self.evictions = 0

    # -- queries ------------------------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free)

    def ref_count(self, block: int) -> int:
        return self.refs[block]

    def block_table(self, seq: int) -> List[int]:
        return list(self.tables[seq])

    def seq_len(self, seq: int) -> int:
        return self.lens[seq]

    # -- mutations ----------------------------------------------------------------------
    def _pop(self) -> int:
        b = self.free.popleft()
        if b in self.block_hash:                 # handed out again: evict its entry
            del self.cache[self.block_hash.pop(b)]
            self.evictions += 1
        self.refs[b] = 1
        return b

    @staticmethod
    def chain_hash(parent: Optional[bytes], tokens: Sequence[int]) -> bytes:
        m = hashlib.sha256()
        if parent is not None:
            m.update(parent)
        m.update(np.asarray(tokens, dtype="<i4").tobytes())
        return m.digest()

    def add_seq_tokens(self, seq: int, tokens: Sequence[int]) -> Tuple[np.ndarray, int]:
        if seq in self.tables:
            raise InvalidCall("add_seq_tokens")
        B = self.block_size
        n = len(tokens)
        nfull, nblk = n // B, -(-n // B)
        hashes: List[bytes] = []
        hits: List[int] = []
        for i in range(nfull):
            hashes.append(self.chain_hash(hashes[-1] if i else None, tokens[i * B:(i + 1) * B]))
            if len(hits) == i and hashes[i] in self.cache:
                hits.append(self.cache[hashes[i]])
        waiting = sum(1 for b in hits if self.refs[b] == 0)
        if nblk - len(hits) > len(self.free) - waiting:
            raise NoBlocks()
        row = []
        for b in hits:
            if self.refs[b] == 0:
                self.free.remove(b)
            self.refs[b] += 1
            row.append(b)
        for i in range(len(hits), nblk):
            b = self._pop()
            row.append(b)
            if i < nfull:
                self.cache[hashes[i]] = b
                self.block_hash[b] = hashes[i]
        self.hit_blocks += len(hits)
        self.tables[seq] = row
        self.lens[seq] = n
        return self._slots(seq, 0, n), len(hits) * B

    def _slots(self, seq: int, start: int, n: int) -> np.ndarray:
        row = self.tables[seq]
        return np.array([slot_of(row, p, self.block_size) for p in range(start, start + n)],
                        dtype=np.int64)

    def add_seq(self, seq: int, num_tokens: int) -> np.ndarray:
        if seq in self.tables or num_tokens < 0:
            raise InvalidCall("add_seq")
        need = -(-num_tokens // self.block_size)
        if need > len(self.free):
            raise NoBlocks()
        self.tables[seq] = [self._pop() for _ in range(need)]
        self.lens[seq] = num_tokens
        return self._slots(seq, 0, num_tokens)

    def fork(self, parent: int, child: int) -> None:
        if parent not in self.tables or child in self.tables:
            raise InvalidCall("fork")
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.refs[b] += 1

    def append(self, seq: int, num_tokens: int) -> Tuple[np.ndarray, List[Tuple[int, int]]]:
        if seq not in self.tables or num_tokens < 0:
            raise InvalidCall("append")
        B = self.block_size
        L = self.lens[seq]
        row = self.tables[seq]
        cow = num_tokens > 0 and L % B != 0 and self.refs[row[-1]] > 1
        grow = -(-(L + num_tokens) // B) - -(-L // B)
        if int(cow) + grow > len(self.free):
            raise NoBlocks()
        pairs: List[Tuple[int, int]] = []
        if cow:
            old = row[-1]
            new = self._pop()
            self.refs[old] -= 1
            row[-1] = new
            pairs.append((old, new))
        for _ in range(grow):
            row.append(self._pop())
        self.lens[seq] = L + num_tokens
        return self._slots(seq, L, num_tokens), pairs

    def append_batch(self, seqs: Sequence[int], counts: Sequence[int]
                     ) -> Tuple[np.ndarray, List[Tuple[int, int]]]:
        """append(seqs[i], counts[i]) for every i, in order, as one all-or-nothing call: the
        policy's "a failed call changes nothing" read for a batch. Ids must be distinct and
        known. Returns the slots of all tokens (sequence after sequence) and the copy pairs
        in batch order."""
        seqs, counts = [int(x) for x in seqs], [int(x) for x in counts]
        if len(seqs) != len(counts) or len(set(seqs)) != len(seqs) or \
                any(s not in self.tables for s in seqs) or any(c < 0 for c in counts):
            raise InvalidCall("append_batch")
        saved = copy.deepcopy(self.__dict__)
        slots, pairs = [], []
        try:
            for s, c in zip(seqs, counts):
                sl, pr = self.append(s, c)
                slots.append(sl)
                pairs.extend(pr)
        except NoBlocks:
            self.__dict__.clear()
            self.__dict__.update(saved)
            raise
        return (np.concatenate(slots) if slots else np.zeros(0, np.int64)), pairs

    def free_seq(self, seq: int) -> None:
        if seq not in self.tables:
            raise InvalidCall("free_seq")
        for b in self.tables.pop(seq):
            self.refs[b] -= 1
            if self.refs[b] == 0:
                self.free.append(b)
        del self.lens[seq]

    def padded_tables(self, seqs: Sequence[int], max_blocks: int) -> np.ndarray:
        """int32 [len(seqs), max_blocks] block tables, unused entries -1."""
        out = np.full((len(seqs), max_blocks), -1, dtype=np.int32)
        for i, s in enumerate(seqs):
            row = self.tables[s]
            out[i, :len(row)] = row
        return out


# ---------------------------------------------------------------------------------------
# cache storage
# ---------------------------------------------------------------------------------------
_STORE = {"f32": np.float32, "bf16": np.uint16, "fp8": np.uint8, "int8": np.int8}


def new_cache(num_blocks: int, num_kv_heads: int, block_size: int, head_dim: int,
              cache_dtype: str) -> np.ndarray:
    """A zeroed cache of storage codes (zeros decode to +0.0 in every format)."""
    return np.zeros((num_blocks, num_kv_heads, block_size, head_dim), dtype=_STORE[cache_dtype])


def _to_f32(x: np.ndarray, in_dtype: str) -> np.ndarray:
    if in_dtype == "f32":
        return np.asarray(x, dtype=np.float32)
    if in_dtype == "bf16":
        return bf16_decode(x).astype(np.float32)  # exact
    raise ValueError(in_dtype)


def _convert(xf: np.ndarray, cache_dtype: str, scale: Optional[np.ndarray],
             zero: Optional[np.ndarray] = None) -> np.ndarray:
    """float32 values -> storage codes of ``cache_dtype``.

    fp8: code = E4M3(x / scale) with the division done in IEEE float32 (round to nearest),
    ``scale`` broadcast over the head dimension. int8: code = clip(rint(x / scale) + zero,
    -128, 127), same division."""
    if cache_dtype == "f32":
        return xf.astype(np.float32)
    if cache_dtype == "bf16":
        return bf16_encode(xf)
    if cache_dtype == "fp8":
        y = (xf / scale[..., None].astype(np.float32)).astype(np.float32)
        return e4m3_encode(y)
    if cache_dtype == "int8":
        y = (xf / scale[..., None].astype(np.float32)).astype(np.float32)
        return int8_encode(y, np.asarray(zero)[..., None])
    raise ValueError(cache_dtype)


def ref_reshape_and_cache(k: np.ndarray, v: np.ndarray, k_cache: np.ndarray,
                          v_cache: np.ndarray, slot_mapping: np.ndarray, in_dtype: str,
                          cache_dtype: str, k_scales: Optional[np.ndarray] = None,
                          v_scales: Optional[np.ndarray] = None,
                          k_zeros: Optional[np.ndarray] = None,
                          v_zeros: Optional[np.ndarray] = None) -> None:
    """Slot-mapped write of new tokens' K and V into the paged cache (in place).

    For token t with slot = slot_mapping[t] >= 0: block = slot // B, offset = slot % B and
    ``cache[block][h][offset][:] = convert(x[t][h][:])`` for every kv head h. A negative
    slot marks a padding token and is skipped. fp8 caches use the per-(block, kv head)
    scale of the destination block; int8 caches its scale and zero point.
    """
    B = k_cache.shape[2]
    slots = np.asarray(slot_mapping, dtype=np.int64)
    for t, slot in enumerate(slots):
        if slot < 0:
            continue
        blk, off = int(slot // B), int(slot % B)
        for x, cache, sc, zp in ((k, k_cache, k_scales, k_zeros), (v, v_cache, v_scales, v_zeros)):
            xf = _to_f32(x[t], in_dtype)  # [Hkv, d]
            s = None if sc is None else sc[blk]  # [Hkv]
            z = None if zp is None else zp[blk]
            cache[blk, :, off, :] = _convert(xf, cache_dtype, s, z)


def ref_copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray,
                    pairs: Sequence[Tuple[int, int]],
                    k_scales: Optional[np.ndarray] = None,
                    v_scales: Optional[np.ndarray] = None,
                    k_zeros: Optional[np.ndarray] = None,
                    v_zeros: Optional[np.ndarray] = None) -> None:
    """Copy-on-write block copy: for each (src, dst) pair, in order, the K and V tiles of
    every kv head (and the quantisation scales / zero points, when given) of ``src`` are
    copied to ``dst``."""
    for src, dst in pairs:
        k_cache[dst] = k_cache[src]
        v_cache[dst] = v_cache[src]
        for arr in (k_scales, v_scales, k_zeros, v_zeros):
            if arr is not None:
                arr[dst] = arr[src]
