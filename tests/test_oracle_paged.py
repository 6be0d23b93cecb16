"""Pins of the oracle's allocator, slot mapping, cache write and block copy.

Against: the pages' block-table example and Theorem 1 (blocks = ceil(T/16), slack <= 15),
the prefix-sharing example (79.2 % token savings at R=100, p=200, s=50) with the ref counts
it implies, conservation invariants, and brute-force read-back of written slots.
"""
import numpy as np
import pytest
import torch

from oracle import codecs, facts, paged
from oracle.paged import RefAllocator, NoBlocks, InvalidCall


def check_invariants(a: RefAllocator):
    live = set()
    total_refs = 0
    for s, row in a.tables.items():
        assert len(row) == facts.blocks_for_tokens(a.lens[s], a.block_size)
        live.update(row)
        total_refs += len(row)
    assert sum(a.refs) == total_refs
    assert len(live) + a.num_free() == a.num_blocks
    assert set(a.free).isdisjoint(live)
    for b in range(a.num_blocks):
        assert (a.refs[b] == 0) == (b not in live)


def test_block_table_example_and_slots(golden):
    g = golden("block_table_example.json")
    a = RefAllocator(8, g["block_size"])
    for i, r in enumerate(g["requests"]):
        slots = a.add_seq(i, r["tokens"])
        row = a.block_table(i)
        assert len(row) == r["blocks"]
        # slot = physical block * B + offset, tokens fill blocks in logical order
        for p, sl in enumerate(slots):
            assert sl == row[p // 16] * 16 + p % 16
        fills = [int(np.sum(slots // 16 == b)) for b in row]
        assert fills == r["fills"]
    check_invariants(a)


@pytest.mark.parametrize("B", [16, 8, 32])
def test_theorem1_slack_on_growth(B):
    a = RefAllocator(65536 // B, B)
    rng = np.random.default_rng(3)
    lens = rng.integers(1, 3000, 40)
    for s, n in enumerate(lens):
        a.add_seq(s, int(n) // 2)
        a.append(s, int(n) - int(n) // 2)
        assert len(a.block_table(s)) == -(-int(n) // B)
        assert len(a.block_table(s)) * B - int(n) <= B - 1
    check_invariants(a)


def test_fifo_order_and_pool_order():
    a = RefAllocator(6, 16, order=[5, 3, 1, 0, 2, 4])
    a.add_seq(0, 20)
    assert a.block_table(0) == [5, 3]
    a.add_seq(1, 1)
    assert a.block_table(1) == [1]
    a.free_seq(0)
    assert list(a.free) == [0, 2, 4, 5, 3]      # freed blocks go to the back, in table order
    with pytest.raises(InvalidCall):
        RefAllocator(3, 16, order=[0, 0, 1])


def test_shortage_is_atomic():
    a = RefAllocator(4, 16)
    a.add_seq(0, 40)           # 3 blocks
    before = (list(a.free), list(a.refs), {k: list(v) for k, v in a.tables.items()}, dict(a.lens))
    with pytest.raises(NoBlocks):
        a.add_seq(1, 17)       # needs 2, 1 free
    with pytest.raises(NoBlocks):
        a.append(0, 30)        # 70 tokens need 5 blocks, has 3, 1 free
    a.fork(0, 2)
    with pytest.raises(NoBlocks):
        a.append(2, 25)        # CoW of the shared partial block + 1 new block: 2 > 1 free
    after = (list(a.free), [r for r in a.refs], {k: list(v) for k, v in a.tables.items() if k != 2},
             {k: v for k, v in a.lens.items() if k != 2})
    assert after[0] == before[0]
    assert after[2] == before[2] and after[3] == before[3]
    with pytest.raises(InvalidCall):
        a.add_seq(0, 1)
    with pytest.raises(InvalidCall):
        a.free_seq(99)
    check_invariants(a)


def test_shared_prefix_example_counts(golden):
    """100 sequences, 200-token shared prefix, 50 private tokens each."""
    g = golden("prefix_sharing.json")["prefix_and_suffix"]
    R, p, s = g["R"], g["p"], g["s_bar"]
    a = RefAllocator(512, 16)
    a.add_seq(0, p)
    for c in range(1, R):
        a.fork(0, c)
    prefix_blocks = a.block_table(0)
    assert len(prefix_blocks) == 13
    assert all(a.ref_count(b) == R for b in prefix_blocks)
    pairs = []
    for sq in range(R):
        _, pr = a.append(sq, s)
        pairs += pr
    # every sequence but the last copies the shared partial block; the last writes in place
    assert len(pairs) == R - 1
    assert all(src == prefix_blocks[-1] for src, _ in pairs)
    assert a.ref_count(prefix_blocks[-1]) == 1 and a.block_table(R - 1)[12] == prefix_blocks[-1]
    assert all(a.ref_count(b) == R for b in prefix_blocks[:12])
    used = a.num_blocks - a.num_free()
    assert used == 12 + R + 3 * R == 412
    # token-level savings of the pages' formula; block-level savings under copy-on-write
    shared_tokens = p + R * s
    unshared_tokens = R * (p + s)
    assert 1 - shared_tokens / unshared_tokens == pytest.approx(facts.sharing_savings(R, p, s))
    assert round(100 * (1 - shared_tokens / unshared_tokens), 1) == g["printed_percent"]
    assert 1 - used / (R * facts.blocks_for_tokens(p + s)) == pytest.approx(1 - 412 / 1600)
    check_invariants(a)
    for sq in range(R):
        a.free_seq(sq)
    assert a.num_free() == 512 and sum(a.refs) == 0


def test_random_traces_keep_invariants():
    rng = np.random.default_rng(7)
    for trial in range(20):
        a = RefAllocator(int(rng.integers(8, 200)), 16)
        live = []
        nxt = 0
        for _ in range(300):
            op = rng.integers(0, 4)
            try:
                if op == 0 or not live:
                    a.add_seq(nxt, int(rng.integers(0, 100)))
                    live.append(nxt)
                    nxt += 1
                elif op == 1:
                    a.fork(live[rng.integers(len(live))], nxt)
                    live.append(nxt)
                    nxt += 1
                elif op == 2:
                    a.append(live[rng.integers(len(live))], int(rng.integers(0, 40)))
                else:
                    a.free_seq(live.pop(rng.integers(len(live))))
            except NoBlocks:
                pass
            check_invariants(a)


def test_cow_append_keeps_shared_content_semantics():
    """After copy + write, every sequence's logical tokens hold its own values."""
    B, H, d = 16, 2, 8
    a = RefAllocator(16, B)
    kc = paged.new_cache(16, H, B, d, "f32")
    vc = paged.new_cache(16, H, B, d, "f32")
    rng = np.random.default_rng(5)
    pre = rng.standard_normal((20, H, d)).astype(np.float32)
    sl = a.add_seq(0, 20)
    paged.ref_reshape_and_cache(pre, pre, kc, vc, sl, "f32", "f32")
    a.fork(0, 1)
    own = {}
    for s in (0, 1):
        x = rng.standard_normal((7, H, d)).astype(np.float32)
        sl, pr = a.append(s, 7)
        paged.ref_copy_blocks(kc, vc, pr)
        paged.ref_reshape_and_cache(x, x, kc, vc, sl, "f32", "f32")
        own[s] = x
    for s in (0, 1):
        row = a.block_table(s)
        full = np.concatenate([pre, own[s]])
        for t in range(27):
            assert np.array_equal(kc[row[t // B], :, t % B], full[t])


def _nearest_code(y, cache_dt, zero=0):
    """Brute force: the codes whose decoded value is nearest to y (all of them on a tie)."""
    if cache_dt == "fp8":
        vals = codecs.E4M3_TABLE
        cand = [c for c in range(256) if np.isfinite(vals[c]) and bool(c & 0x80) == bool(np.signbit(y))]
        dist = [abs(float(y) - vals[c]) for c in cand]
    else:
        cand = list(range(-128, 128))
        dist = [abs(float(y) - (c - zero)) for c in cand]
    best = min(dist)
    return [c for c, dd in zip(cand, dist) if dd == best]


@pytest.mark.parametrize("in_dt,cache_dt", [("f32", "f32"), ("f32", "bf16"), ("bf16", "bf16"),
                                            ("bf16", "fp8"), ("f32", "fp8"), ("f32", "int8"),
                                            ("bf16", "int8")])
def test_reshape_and_cache_readback(in_dt, cache_dt):
    """K and V get different inputs, scales and zero points; every written element is read
    back against the format's definition (fp8 / int8: a nearest code to x / scale, the int8
    code offset by the block's zero point and clipped to the byte's range)."""
    rng = np.random.default_rng(11)
    NB, H, B, d, T = 10, 3, 16, 16, 37
    quant = cache_dt in ("fp8", "int8")
    big = 40.0 if cache_dt == "int8" else 1.0       # int8: values span many codes and clip
    raw = {n: (rng.standard_normal((T, H, d)) * big).astype(np.float32) for n in "kv"}
    x = {n: raw[n] if in_dt == "f32" else codecs.bf16_encode(raw[n]) for n in "kv"}
    xv = {n: raw[n] if in_dt == "f32" else codecs.bf16_decode(x[n]).astype(np.float32) for n in "kv"}
    slots = rng.permutation(NB * B)[:T].astype(np.int64)
    slots[3] = -1
    sc = {n: rng.uniform(0.5, 2.0, (NB, H)).astype(np.float32) for n in "kv"}
    zp = {n: rng.integers(-40, 41, (NB, H)).astype(np.int32) for n in "kv"}
    cache = {n: paged.new_cache(NB, H, B, d, cache_dt) for n in "kv"}
    paged.ref_reshape_and_cache(x["k"], x["v"], cache["k"], cache["v"], slots, in_dt, cache_dt,
                                sc["k"] if quant else None, sc["v"] if quant else None,
                                zp["k"] if cache_dt == "int8" else None,
                                zp["v"] if cache_dt == "int8" else None)
    written = np.zeros((NB, B), bool)
    for t, sl in enumerate(slots):
        if sl < 0:
            continue
        blk, off = sl // B, sl % B
        written[blk, off] = True
        for n in "kv":
            got = cache[n][blk, :, off, :]
            if cache_dt == "f32":
                assert np.array_equal(got, xv[n][t])
            elif cache_dt == "bf16":
                ref = torch.from_numpy(xv[n][t].copy()).to(torch.bfloat16).view(torch.int16).numpy()
                assert np.array_equal(got, ref.view(np.uint16))
            else:
                y = (xv[n][t] / sc[n][blk][:, None]).astype(np.float32)
                for h in range(H):
                    z = int(zp[n][blk, h]) if cache_dt == "int8" else 0
                    for j in range(d):
                        assert int(got[h, j]) in _nearest_code(y[h, j], cache_dt, z)
    # unwritten slots stay zero
    mask = np.broadcast_to(~written[:, None, :, None], cache["k"].shape)
    assert np.all(cache["k"][mask] == 0) and np.all(cache["v"][mask] == 0)


def test_copy_blocks_copies_tiles_and_scales():
    rng = np.random.default_rng(4)
    NB, H, B, d = 12, 2, 16, 8
    kc = rng.integers(0, 255, (NB, H, B, d)).astype(np.uint8)
    vc = rng.integers(0, 255, (NB, H, B, d)).astype(np.uint8)
    ks = rng.uniform(size=(NB, H)).astype(np.float32)
    vs = rng.uniform(size=(NB, H)).astype(np.float32)
    k0, v0, ks0, vs0 = kc.copy(), vc.copy(), ks.copy(), vs.copy()
    pairs = [(1, 7), (2, 9), (1, 11)]
    paged.ref_copy_blocks(kc, vc, pairs, ks, vs)
    for s, t in pairs:
        assert np.array_equal(kc[t], k0[s]) and np.array_equal(vc[t], v0[s])
        assert ks[t] == pytest.approx(ks0[s]) and np.array_equal(vs[t], vs0[s])
    untouched = [b for b in range(NB) if b not in (7, 9, 11)]
    assert np.array_equal(kc[untouched], k0[untouched]) and np.array_equal(ks[untouched], ks0[untouched])


def test_append_batch_hand_worked_and_all_or_nothing():
    """Three forks share a partially filled last block (ref_count 3). Appending one token to
    each in one batch copies it for the first two (ref 3 -> 2 -> 1); the third then owns it
    and writes in place. A batch one block short changes nothing."""
    B = 16
    a = RefAllocator(8, B)
    a.add_seq(0, 20)                            # blocks 0, 1 (block 1 holds 4 tokens)
    a.fork(0, 1)
    a.fork(0, 2)
    slots, pairs = a.append_batch([1, 2, 0], [1, 1, 1])
    assert pairs == [(1, 2), (1, 3)]            # seq 1 copies into 2, seq 2 into 3
    assert a.block_table(1) == [0, 2] and a.block_table(2) == [0, 3] and a.block_table(0) == [0, 1]
    assert list(slots) == [2 * B + 4, 3 * B + 4, 1 * B + 4]
    assert a.refs[:4] == [3, 1, 1, 1] and list(a.free) == [4, 5, 6, 7]
    # 4 free blocks; seq 0 needs 1 more (to 40 tokens), seqs 1 and 2 two each (to 49): 5 > 4
    snap = (list(a.free), list(a.refs), {s: list(r) for s, r in a.tables.items()}, dict(a.lens))
    with pytest.raises(NoBlocks):
        a.append_batch([0, 1, 2], [19, 28, 28])
    assert snap == (list(a.free), list(a.refs), {s: list(r) for s, r in a.tables.items()},
                    dict(a.lens))
    # without its last member the batch fits (1 + 2 = 3 blocks of 4)
    slots, pairs = a.append_batch([0, 1], [19, 28])
    assert pairs == [] and len(slots) == 47 and a.num_free() == 1
    with pytest.raises(InvalidCall):
        a.append_batch([0, 0], [1, 1])          # duplicate id
    with pytest.raises(InvalidCall):
        a.append_batch([0, 9], [1, 1])          # unknown id
