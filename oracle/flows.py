"""The hot path end to end, oracle side (test infrastructure only).

Runs the steps in the order a decode step takes them — allocation and slot mapping, the
copy-on-write block copies, the slot-mapped cache write, decode attention — on one seeded
draw from ``workloads``. Only oracle functions are called.

Flows (readings of the pages, stated once):
* decode workloads: an allocator whose free queue starts in the draw's pool order; every
  sequence is added with ctx-1 tokens (in sequence order), then every sequence appends its
  decode token (ctx includes the token being decoded); all K/V is written through the
  slot mapping, then attention runs.
* prefill workloads: every sequence is added with its cached tokens (ctx - n), in
  sequence order, then every sequence appends its n new tokens; all K/V is written through
  the slot mapping, then the new tokens attend causally.
* shared-prefix workload ([KVPaged] "Prefix sharing and copy-on-write", [Ch4PA] "Prefix
  Caching"): sequence 0 is added with the prefix and the prefix K/V written once; it is
  forked to every other sequence; every sequence then appends its private suffix in
  sequence order, which copies the shared partial last block first (copy-on-write); the
  copies run before any suffix token is written.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np

from .paged import RefAllocator, new_cache, ref_copy_blocks, ref_reshape_and_cache
from .attention import ref_decode, ref_prefill


@dataclasses.dataclass
class RefState:
    alloc: RefAllocator
    k_cache: np.ndarray
    v_cache: np.ndarray
    k_scales: Optional[np.ndarray]
    v_scales: Optional[np.ndarray]
    block_tables: np.ndarray
    context_lens: np.ndarray
    cow_pairs: List
    step_slots: Dict[int, np.ndarray]
    k_zeros: Optional[np.ndarray] = None
    v_zeros: Optional[np.ndarray] = None


def max_blocks_per_seq(draw) -> int:
    B = draw.wl.block_size
    return int(max(1, -(-int(draw.context_lens.max()) // B)))


def _fp8_scales(draw, alloc, seqs, nb, hkv):
    ks = np.ones((nb, hkv), dtype=np.float32)
    vs = np.ones((nb, hkv), dtype=np.float32)
    for s in seqs:
        lk, lv = draw.fp8_scales_logical(s)
        row = alloc.block_table(s)
        ks[row] = lk
        vs[row] = lv
    return ks, vs


def _int8_params(draw, alloc, seqs, nb, hkv):
    ks = np.ones((nb, hkv), dtype=np.float32)
    vs = np.ones((nb, hkv), dtype=np.float32)
    kz = np.zeros((nb, hkv), dtype=np.int32)
    vz = np.zeros((nb, hkv), dtype=np.int32)
    for s in seqs:
        lks, lkz, lvs, lvz = draw.int8_params_logical(s)
        row = alloc.block_table(s)
        ks[row], kz[row], vs[row], vz[row] = lks, lkz, lvs, lvz
    return ks, vs, kz, vz


def build_state(draw, write_seqs: Optional[Sequence[int]] = None, shared: bool = True) -> RefState:
    """Allocate, copy and write the whole workload. K/V is written only for ``write_seqs``
    (default: all), which bounds the work for large workloads checked on a sample; the
    allocator always sees every sequence, so block placement is the full workload's.
    ``shared=False`` lays a shared-prefix workload out as private, unshared copies."""
    wl = draw.wl
    S, B, H, d = wl.num_seqs, wl.block_size, wl.num_kv_heads, wl.head_dim
    write = set(range(S) if write_seqs is None else write_seqs)
    nb = wl.num_blocks
    if wl.shared_prefix is not None and not shared:
        nb = max(nb, S * max_blocks_per_seq(draw))
    alloc = RefAllocator(nb, B, order=draw.pool_order if nb == wl.num_blocks else None)
    kc = new_cache(nb, H, B, d, wl.kv_dtype)
    vc = new_cache(nb, H, B, d, wl.kv_dtype)
    ks = vs = kz = vz = None
    pairs: List = []
    step_slots: Dict[int, np.ndarray] = {}
    if wl.shared_prefix is not None and shared:
        p, sfx = wl.shared_prefix
        slots0 = alloc.add_seq(0, p)
        for c in range(1, S):
            alloc.fork(0, c)
        sfx_slots = {}
        for s in range(S):
            sl, pr = alloc.append(s, sfx)
            sfx_slots[s] = sl
            pairs += pr
        if wl.kv_dtype == "fp8":
            ks, vs = _fp8_scales(draw, alloc, range(S), nb, H)
        elif wl.kv_dtype == "int8":
            ks, vs, kz, vz = _int8_params(draw, alloc, range(S), nb, H)
        k0, v0 = draw.kv(0)
        ref_reshape_and_cache(k0[:p], v0[:p], kc, vc, slots0, wl.in_dtype, wl.kv_dtype, ks, vs,
                              kz, vz)
        ref_copy_blocks(kc, vc, pairs, ks, vs, kz, vz)
        for s in sorted(write):
            k, v = draw.kv(s)
            ref_reshape_and_cache(k[p:], v[p:], kc, vc, sfx_slots[s], wl.in_dtype, wl.kv_dtype,
                                  ks, vs, kz, vz)
            step_slots[s] = sfx_slots[s]
    else:
        pre = {}
        for s in range(S):
            pre[s] = alloc.add_seq(s, int(draw.context_lens[s]) - 1)
        for s in range(S):
            sl, pr = alloc.append(s, 1)
            assert not pr
            step_slots[s] = sl
        if wl.kv_dtype == "fp8":
            ks, vs = _fp8_scales(draw, alloc, write, nb, H)
        elif wl.kv_dtype == "int8":
            ks, vs, kz, vz = _int8_params(draw, alloc, write, nb, H)
        for s in sorted(write):
            k, v = draw.kv(s)
            ref_reshape_and_cache(k[:-1], v[:-1], kc, vc, pre[s], wl.in_dtype, wl.kv_dtype, ks, vs,
                                  kz, vz)
            ref_reshape_and_cache(k[-1:], v[-1:], kc, vc, step_slots[s], wl.in_dtype,
                                  wl.kv_dtype, ks, vs, kz, vz)
    tables = alloc.padded_tables(range(S), max_blocks_per_seq(draw))
    return RefState(alloc, kc, vc, ks, vs, tables, draw.context_lens.copy(), pairs, step_slots,
                    kz, vz)


def ref_outputs(draw, state: RefState, seqs: Optional[Sequence[int]] = None, scale=None):
    wl = draw.wl
    # the scale is a float32 argument of the kernel; the oracle uses that same value
    sc = float(np.float32(1.0 / np.sqrt(wl.head_dim) if scale is None else scale))
    return ref_decode(draw.q, state.k_cache, state.v_cache, state.block_tables,
                      state.context_lens, sc, wl.num_kv_heads, wl.in_dtype, wl.kv_dtype,
                      state.k_scales, state.v_scales, seqs=seqs, k_zeros=state.k_zeros,
                      v_zeros=state.v_zeros)


def build_prefill_state(draw, write_seqs: Optional[Sequence[int]] = None) -> RefState:
    """Allocate and write a prefill step: cached tokens first (add_seq), then the step's
    new tokens (append); K/V written only for ``write_seqs`` (default all)."""
    wl = draw.wl
    S, B, H, d = wl.num_seqs, wl.block_size, wl.num_kv_heads, wl.head_dim
    write = set(range(S) if write_seqs is None else write_seqs)
    nb = wl.num_blocks
    alloc = RefAllocator(nb, B, order=draw.pool_order)
    kc = new_cache(nb, H, B, d, wl.kv_dtype)
    vc = new_cache(nb, H, B, d, wl.kv_dtype)
    ks = vs = kz = vz = None
    pre, new = {}, {}
    for s in range(S):
        pre[s] = alloc.add_seq(s, int(draw.context_lens[s] - draw.query_lens[s]))
    for s in range(S):
        sl, pr = alloc.append(s, int(draw.query_lens[s]))
        assert not pr
        new[s] = sl
    if wl.kv_dtype == "fp8":
        ks, vs = _fp8_scales(draw, alloc, write, nb, H)
    elif wl.kv_dtype == "int8":
        ks, vs, kz, vz = _int8_params(draw, alloc, write, nb, H)
    for s in sorted(write):
        k, v = draw.kv(s)
        c = int(draw.context_lens[s] - draw.query_lens[s])
        ref_reshape_and_cache(k[:c], v[:c], kc, vc, pre[s], wl.in_dtype, wl.kv_dtype, ks, vs,
                              kz, vz)
        ref_reshape_and_cache(k[c:], v[c:], kc, vc, new[s], wl.in_dtype, wl.kv_dtype, ks, vs,
                              kz, vz)
    tables = alloc.padded_tables(range(S), max_blocks_per_seq(draw))
    return RefState(alloc, kc, vc, ks, vs, tables, draw.context_lens.copy(), [], new, kz, vz)


def ref_prefill_outputs(draw, state: RefState, seqs: Optional[Sequence[int]] = None,
                        scale=None):
    wl = draw.wl
    sc = float(np.float32(1.0 / np.sqrt(wl.head_dim) if scale is None else scale))
    return ref_prefill(draw.q, draw.query_start, state.k_cache, state.v_cache,
                       state.block_tables, state.context_lens, sc, wl.num_kv_heads,
                       wl.in_dtype, wl.kv_dtype, state.k_scales, state.v_scales,
                       state.k_zeros, state.v_zeros, seqs=seqs)
