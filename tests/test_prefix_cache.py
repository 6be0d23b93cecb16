"""Automatic prefix caching in the native allocator.

CPU: the library's SHA-256 against hashlib; chained block hashes and the whole allocator
state (free queue order, ref counts, tables, cache entries, hit / eviction totals) equal to
the oracle's on random traces; the shared-system-prompt example reproduces the pages'
savings formula for the block-aligned part of the prompt; LRU eviction order; atomic
failure. GPU: decode over a prefix-cached layout (cached blocks written once) equals the
decode over private copies, bit for bit.
"""
import hashlib

import numpy as np
import pytest

from oracle import facts
from oracle.paged import RefAllocator, NoBlocks as RefNoBlocks, InvalidCall


@pytest.fixture(scope="module")
def pa():
    import importlib.util
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location(
        "_pa_build", os.path.join(root, "paged_kv_cache_465_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import paged_kv_cache_465_b200 as pa
    return pa


def test_sha256_matches_hashlib(pa):
    rng = np.random.default_rng(0)
    for n in list(range(0, 130)) + [1000, 4096, 10007]:
        m = rng.integers(0, 256, n, dtype=np.uint8).tobytes()
        assert pa.sha256(m) == hashlib.sha256(m).digest(), n


def _state(nat, ref):
    assert nat.free_queue() == list(ref.free)
    assert [nat.ref_count(b) for b in range(ref.num_blocks)] == ref.refs
    assert nat.num_cached() == len(ref.cache)
    assert nat.cache_stats() == (ref.hit_blocks, ref.evictions)
    for b in range(ref.num_blocks):
        assert nat.block_hash(b) == ref.block_hash.get(b)


def test_chained_hashes_and_random_traces_match_oracle(pa):
    rng = np.random.default_rng(1)
    prompts = [rng.integers(0, 50000, int(rng.integers(0, 90))).tolist() for _ in range(6)]
    for trial in range(12):
        nb = int(rng.integers(6, 120))
        order = rng.permutation(nb) if trial % 2 else None
        ref = RefAllocator(nb, 16, order=order)
        nat = pa.BlockAllocator(nb, 16, order=order)
        live, nxt = [], 0
        for step in range(250):
            op = int(rng.integers(0, 6))
            if op <= 1 or not live:
                base = prompts[int(rng.integers(len(prompts)))]
                cut = int(rng.integers(0, len(base) + 1))
                toks = base[:cut] + rng.integers(0, 50000, int(rng.integers(0, 40))).tolist()
                args = ("add_seq_tokens", nxt, toks)
            elif op == 2:
                args = ("fork", live[int(rng.integers(len(live)))], nxt)
            elif op == 3:
                args = ("append", live[int(rng.integers(len(live)))], int(rng.integers(0, 30)))
            else:
                args = ("free_seq", live[int(rng.integers(len(live)))])
            r_exc = n_exc = None
            try:
                r_res = getattr(ref, args[0])(*args[1:])
            except (RefNoBlocks, InvalidCall) as e:
                r_exc = type(e).__name__
            try:
                n_res = getattr(nat, args[0])(*args[1:])
            except pa.NoBlocks:
                n_exc = "NoBlocks"
            except pa.PagedAttnError:
                n_exc = "InvalidCall"
            assert r_exc == n_exc, (args[0], r_exc, n_exc)
            if r_exc is None:
                if args[0] in ("add_seq_tokens", "fork"):
                    live.append(args[1] if args[0] == "add_seq_tokens" else args[2])
                    nxt += 1
                if args[0] == "free_seq":
                    live.remove(args[1])
                if args[0] == "add_seq_tokens":
                    assert np.array_equal(r_res[0], n_res[0]) and r_res[1] == n_res[1]
            _state(nat, ref)
            for s in live:
                assert nat.block_table(s) == ref.block_table(s)


def test_shared_system_prompt_savings(pa):
    """100 requests, a common 200-token prompt, 50 private tokens each."""
    R, p, sfx, B = 100, 200, 50, 16
    rng = np.random.default_rng(2)
    prompt = rng.integers(0, 32000, p).tolist()
    a = pa.BlockAllocator(512, B)
    cached = []
    for r in range(R):
        toks = prompt + rng.integers(0, 32000, sfx).tolist()
        _, c = a.add_seq_tokens(r, toks)
        cached.append(c)
    assert cached[0] == 0 and all(c == (p // B) * B for c in cached[1:])   # 12 full blocks
    assert 512 - a.num_free() == 16 + (R - 1) * (16 - 12) == 412
    reused = sum(cached)
    # the pages' (R-1) p / (R (p + s)) with the block-aligned prompt p = 192
    assert reused / (R * (p + sfx)) == pytest.approx(facts.sharing_savings(R, 192, p + sfx - 192))
    assert a.cache_stats() == ((R - 1) * 12, 0)


def test_lru_eviction_order(pa):
    B = 16
    a = pa.BlockAllocator(8, B)
    x = list(range(1, 33))      # 2 full blocks
    y = list(range(100, 132))   # 2 full blocks
    a.add_seq_tokens(0, x)
    a.add_seq_tokens(1, y)
    bx, by = a.block_table(0), a.block_table(1)
    a.free_seq(0)               # x's blocks wait first (least recently used) ...
    a.free_seq(1)               # ... then y's
    assert a.num_cached() == 4 and a.num_free() == 8
    a.add_seq(2, 4 * B)         # pops the 4 never-used blocks
    plain = a.block_table(2)
    a.add_seq(3, 2 * B)         # pops x's two blocks: their entries are evicted
    assert a.block_table(3) == bx and a.cache_stats()[1] == 2
    a.free_seq(2)               # queue: y's blocks, then the 4 plain ones
    assert a.free_queue() == by + plain
    _, c = a.add_seq_tokens(5, y + [7])
    assert c == 32 and a.block_table(5) == by + plain[:1]   # y reused from the queue
    _, c = a.add_seq_tokens(4, x)
    assert c == 0 and a.block_table(4) == plain[1:3]       # x was evicted


def test_shortage_with_hits_is_atomic(pa):
    a = pa.BlockAllocator(4, 16)
    p = list(range(48))         # 3 full blocks
    a.add_seq_tokens(0, p)
    a.free_seq(0)
    a.add_seq(1, 16)            # 3 cached blocks wait, 0 plain free... the queue holds 3
    before = (a.free_queue(), a.num_cached(), a.cache_stats())
    with pytest.raises(pa.NoBlocks):
        a.add_seq_tokens(2, p + list(range(100, 140)))   # 3 hits + 3 new blocks > 3 free - 3 hits
    assert (a.free_queue(), a.num_cached(), a.cache_stats()) == before
    _, c = a.add_seq_tokens(3, p)
    assert c == 48 and a.num_free() == 0


@pytest.mark.gpu
def test_prefix_cached_decode_matches_private_copies(pa):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_465_b200.cache import PagedKVCache
    rng = np.random.default_rng(3)
    H, Hq, d, B = 8, 32, 128, 16
    prompt = rng.integers(0, 32000, 333).tolist()
    seqs = [prompt + rng.integers(0, 32000, n).tolist() for n in (1, 77, 300)]
    # per-token K/V is a function of the token prefix: identical prompts -> identical K/V
    kv = {}
    gen = torch.Generator().manual_seed(4)
    table_k = torch.randn(len(prompt) + 301, H, d, generator=gen).to(torch.bfloat16)
    table_v = torch.randn(len(prompt) + 301, H, d, generator=gen).to(torch.bfloat16)
    priv_k = [torch.randn(len(s), H, d, generator=gen).to(torch.bfloat16) for s in seqs]
    priv_v = [torch.randn(len(s), H, d, generator=gen).to(torch.bfloat16) for s in seqs]
    for i, s in enumerate(seqs):
        kv[i] = (torch.cat([table_k[:len(prompt)], priv_k[i][len(prompt):]]).cuda(),
                 torch.cat([table_v[:len(prompt)], priv_v[i][len(prompt):]]).cuda())
    q = torch.randn(len(seqs), Hq, d, generator=gen).to(torch.bfloat16).cuda()
    lens = torch.tensor([len(s) for s in seqs], dtype=torch.int32).cuda()
    mb = max(-(-len(s) // B) for s in seqs)
    outs = []
    for cached_mode in (True, False):
        c = PagedKVCache(256, H, d, "bf16", B)
        written = 0
        for i, s in enumerate(seqs):
            if cached_mode:
                slots, ncached = c.alloc.add_seq_tokens(i, s)
            else:
                slots, ncached = c.add_seq(i, len(s)), 0
            k, v = kv[i]
            sl = torch.from_numpy(slots[ncached:]).cuda()
            c.write(k[ncached:].contiguous(), v[ncached:].contiguous(), sl)
            written += len(s) - ncached
        bt = c.block_tables(range(len(seqs)), mb).cuda()
        out = torch.empty_like(q)
        ws = torch.empty(1 << 22, dtype=torch.uint8, device="cuda")
        c.decode(q, bt, lens, 0.0883883, out, max_context_len=int(lens.max()), partition_size=256,
                 workspace=ws)
        torch.cuda.synchronize()
        assert pa.device_error() == 0
        outs.append((out, written))
    (o1, w1), (o2, w2) = outs
    assert w1 == w2 - 2 * (len(prompt) // B) * B     # two hits on 20 cached prompt blocks
    assert torch.equal(o1, o2)
