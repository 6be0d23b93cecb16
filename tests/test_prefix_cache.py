"""Automatic prefix caching in the native allocator.

CPU: the library's SHA-256 against hashlib; chained block hashes and the whole allocator
state (free queue order, ref counts, tables, cache entries, hit / eviction totals) equal to
the oracle's on random traces; the shared-system-prompt example reproduces the pages'
savings formula for the block-aligned part of the prompt; LRU eviction order; atomic
failure. GPU: the prefix-cached flow (add_seq_tokens, writes of the uncached tokens only,
prefill over a prefix hit, decode, frees, hits on freed blocks, evictions) through the
library equals the oracle's flow (allocator state and cache bytes bit for bit, attention
within tolerance); decode over a prefix-cached layout (cached blocks written once) equals
the decode over private copies, bit for bit.
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


# ---------------------------------------------------------------------------------------
# GPU: the prefix-cached flow through the library against the oracle's flow
# ---------------------------------------------------------------------------------------
def _token_kv(tokens, H, d):
    """K and V [n, H, d] float32 of a token list, token p's depending on tokens[0..p] only
    (a stand-in for a model layer): requests with a common prefix get equal prefix K/V, as
    the pages' prefix caching assumes ([KVPaged] "Prefix cache lifetime and invalidation":
    a hit reuses the cached prefix KV instead of recomputing it)."""
    key = b""
    ks, vs = [], []
    for t in tokens:
        key = hashlib.sha256(key + int(t).to_bytes(4, "little", signed=True)).digest()
        rng = np.random.default_rng(int.from_bytes(key[:8], "little"))
        ks.append(rng.standard_normal((H, d), dtype=np.float32))
        vs.append(rng.standard_normal((H, d), dtype=np.float32))
    return np.stack(ks), np.stack(vs)


def _bf16_values(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32)


class _PrefixFlow:
    """One pool driven twice from the same requests: through the library (native allocator
    with prefix caching, cache write, prefill and decode kernels) and through the oracle
    (RefAllocator.add_seq_tokens, ref_reshape_and_cache, ref_prefill, ref_decode).

    fp8 block scales are set when a block is first filled: absmax / 448 of the tokens that
    fill it then; tokens written into it later keep that scale (they saturate at +-448 if
    larger), on both sides alike. A block reused by a cache hit keeps its scale."""

    def __init__(self, pa, torch, kv_dtype, NB=64, H=8, Hq=32, d=128, B=16, seed=31):
        from oracle import paged as opaged
        from paged_kv_cache_465_b200.cache import PagedKVCache
        self.pa, self.torch, self.kv_dtype = pa, torch, kv_dtype
        self.H, self.Hq, self.d, self.B, self.NB = H, Hq, d, B, NB
        self.rng = np.random.default_rng(seed)
        order = self.rng.permutation(NB).astype(np.int32)
        self.ref = RefAllocator(NB, B, order=order)
        self.gpu = PagedKVCache(NB, H, d, kv_dtype, B, order=order)
        self.kc = opaged.new_cache(NB, H, B, d, kv_dtype)
        self.vc = opaged.new_cache(NB, H, B, d, kv_dtype)
        quant = kv_dtype == "fp8"
        self.ks = np.ones((NB, H), np.float32) if quant else None
        self.vs = np.ones((NB, H), np.float32) if quant else None
        self.fresh = set()  # blocks popped for new content whose scale is not set yet
        self.tokens = {}    # seq -> token ids (including appended decode tokens)
        self.kv = {}        # seq -> (K, V) bf16 bits of every token

    def to_dev(self, bits):
        t = self.torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
        return t.view(self.torch.bfloat16).cuda()

    def set_kv(self, s):
        import workloads
        K, V = _token_kv(self.tokens[s], self.H, self.d)
        self.kv[s] = (workloads.bf16_bits_from_f32(K), workloads.bf16_bits_from_f32(V))

    def set_scales(self, seqs):
        if self.ks is None:
            return
        B = self.B
        for s in seqs:
            n = len(self.tokens[s])
            for i, b in enumerate(self.ref.block_table(s)):
                if b not in self.fresh:
                    continue
                self.fresh.discard(b)
                for x, sc in zip(self.kv[s], (self.ks, self.vs)):
                    am = np.abs(_bf16_values(x[i * B:min(n, (i + 1) * B)])).max(axis=(0, 2))
                    sc[b] = np.where(am > 0, am / np.float32(448.0), 1.0).astype(np.float32)
        self.gpu.k_scales.copy_(self.torch.from_numpy(self.ks))
        self.gpu.v_scales.copy_(self.torch.from_numpy(self.vs))

    def add(self, seq, toks):
        """add_seq_tokens on both sides: (slots, cached leading tokens)."""
        r_slots, r_cached = self.ref.add_seq_tokens(seq, toks)
        g_slots, g_cached = self.gpu.alloc.add_seq_tokens(seq, toks)
        assert np.array_equal(r_slots, g_slots) and r_cached == g_cached
        self.fresh.update(self.ref.block_table(seq)[r_cached // self.B:])
        self.tokens[seq] = list(toks)
        self.set_kv(seq)
        return r_slots, r_cached

    def write(self, items):
        """items: (seq, first position, slots): that sequence's K/V from that position on,
        written on both sides."""
        from oracle import paged as opaged
        for s, p0, slots in items:
            kb, vb = self.kv[s][0][p0:], self.kv[s][1][p0:]
            opaged.ref_reshape_and_cache(kb, vb, self.kc, self.vc, slots, "bf16", self.kv_dtype,
                                         self.ks, self.vs)
            if len(slots):
                self.gpu.write(self.to_dev(kb), self.to_dev(vb),
                               self.torch.from_numpy(np.asarray(slots, np.int64)).cuda())
        self.torch.cuda.synchronize()
        assert self.pa.device_error() == 0

    def check_state(self):
        from gpu_common import cache_codes
        assert self.gpu.alloc.free_queue() == list(self.ref.free)
        assert [self.gpu.alloc.ref_count(b) for b in range(self.NB)] == self.ref.refs
        assert self.gpu.alloc.num_cached() == len(self.ref.cache)
        assert self.gpu.alloc.cache_stats() == (self.ref.hit_blocks, self.ref.evictions)
        for b in range(self.NB):
            assert self.gpu.alloc.block_hash(b) == self.ref.block_hash.get(b)
        for s in self.tokens:
            assert self.gpu.alloc.block_table(s) == self.ref.block_table(s)
        assert np.array_equal(cache_codes(self.gpu.k_cache), self.kc)
        assert np.array_equal(cache_codes(self.gpu.v_cache), self.vc)

    def tables(self, seqs):
        mb = max(len(self.ref.block_table(s)) for s in seqs)
        return self.ref.padded_tables(seqs, mb)


@pytest.mark.gpu
@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_prefix_cache_flow_matches_oracle(pa, kv_dtype):
    """Requests sharing a 200-token system prompt (12 full blocks), one that is exactly the
    cached part, one that extends an earlier request, and an unrelated one go through
    add_seq_tokens; only the uncached tokens are written and attend (prefill); a decode
    token is appended to every live request and decoded in 64-token partitions; then two
    requests are freed, a repeat of one of them reuses its blocks and a long new request
    pops the free queue down to cached blocks (evictions). At every stage the allocator
    state (slots, cached-token counts, tables, ref counts, free queue, cache entries and
    hashes, hit / eviction totals) and every cache byte equal the oracle's, and prefill and
    decode outputs match the oracle within the storage type's tolerances."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import workloads
    from oracle import attention
    from gpu_common import compare_decode
    f = _PrefixFlow(pa, torch, kv_dtype)
    rng = f.rng
    scale = float(np.float32(1.0 / np.sqrt(f.d)))

    def qdraw(n):
        return workloads.bf16_bits_from_f32(rng.standard_normal((n, f.Hq, f.d), dtype=np.float32))

    def prefill(new):
        """new: seq -> (slots, cached) of freshly added requests. Writes the uncached
        tokens, then runs prefill over them on both sides and compares."""
        seqs = sorted(new)
        f.set_scales(seqs)
        f.write([(s, new[s][1], new[s][0][new[s][1]:]) for s in seqs])
        f.check_state()
        n = [len(f.tokens[s]) - new[s][1] for s in seqs]
        qs = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
        T = int(qs[-1])
        qb = qdraw(T)
        ctx = np.array([len(f.tokens[s]) for s in seqs], np.int32)
        bt = f.tables(seqs)
        ref_o, ref_l = attention.ref_prefill(qb, qs, f.kc, f.vc, bt, ctx, scale, f.H, "bf16",
                                             kv_dtype, f.ks, f.vs)
        out = torch.empty((T, f.Hq, f.d), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((T, f.Hq), dtype=torch.float32, device="cuda")
        f.gpu.prefill(f.to_dev(qb), torch.from_numpy(bt).cuda(), torch.from_numpy(ctx).cuda(),
                      torch.from_numpy(qs).cuda(), scale, out, max_query_len=max(n),
                      max_context_len=int(ctx.max()), lse_out=lse)
        torch.cuda.synchronize()
        assert pa.device_error() == 0
        compare_decode(out, lse, ref_o, ref_l, kv_dtype)
        return n

    prompt = rng.integers(0, 32000, 200).tolist()
    r0 = prompt + rng.integers(0, 32000, 50).tolist()
    reqs = {0: r0,
            1: prompt + rng.integers(0, 32000, 30).tolist(),
            2: prompt[:192],                                   # exactly the cached blocks
            3: r0 + rng.integers(0, 32000, 40).tolist(),       # extends request 0
            4: rng.integers(0, 32000, 77).tolist()}            # unrelated
    new = {s: f.add(s, toks) for s, toks in reqs.items()}
    assert {s: new[s][1] for s in new} == {0: 0, 1: 192, 2: 192, 3: 240, 4: 0}
    assert prefill(new) == [250, 38, 0, 50, 77]     # only the uncached tokens attend

    # decode: one new token for every live request, split into 64-token partitions
    live = sorted(f.tokens)
    r_slots, r_pairs = f.ref.append_batch(live, [1] * len(live))
    g_slots, g_pairs = f.gpu.alloc.append_batch(live, 1)
    assert np.array_equal(r_slots, g_slots) and len(r_pairs) == 0 and len(g_pairs) == 0
    for s, t in zip(live, rng.integers(0, 32000, len(live)).tolist()):
        f.tokens[s].append(t)
        f.set_kv(s)
        if (len(f.tokens[s]) - 1) % f.B == 0:      # the token opened a new block
            f.fresh.add(f.ref.block_table(s)[-1])
    f.set_scales(live)
    f.write([(s, len(f.tokens[s]) - 1, r_slots[i:i + 1]) for i, s in enumerate(live)])
    f.check_state()
    qb = qdraw(len(live))
    ctx = np.array([len(f.tokens[s]) for s in live], np.int32)
    bt = f.tables(live)
    ref_o, ref_l = attention.ref_decode(qb, f.kc, f.vc, bt, ctx, scale, f.H, "bf16", kv_dtype,
                                        f.ks, f.vs)
    out = torch.empty((len(live), f.Hq, f.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((len(live), f.Hq), dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 22, dtype=torch.uint8, device="cuda")
    f.gpu.decode(f.to_dev(qb), torch.from_numpy(bt).cuda(), torch.from_numpy(ctx).cuda(), scale,
                 out, max_context_len=int(ctx.max()), partition_size=64, lse_out=lse, workspace=ws)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    compare_decode(out, lse, ref_o, ref_l, kv_dtype)

    # free two requests; a repeat of request 0 reuses its 15 full blocks, a 600-token new
    # request pops the free queue past request 4's cached blocks (evicting them)
    for s in (0, 4):
        f.ref.free_seq(s)
        f.gpu.alloc.free_seq(s)
        del f.tokens[s], f.kv[s]
    f.check_state()
    hits0, ev0 = f.ref.hit_blocks, f.ref.evictions
    new = {5: f.add(5, r0), 6: f.add(6, rng.integers(0, 32000, 600).tolist())}
    assert new[5][1] == 240 and new[6][1] == 0
    assert f.ref.hit_blocks - hits0 == 15 and f.ref.evictions - ev0 == 3
    assert prefill(new) == [10, 600]
