"""CPU checks of the native library: it builds, loads and exports every symbol the header
declares; its host allocator matches the oracle's allocator state bit for bit on random
traces and on the shared-prefix example; host-side validation rejects bad calls before any
device work (none of these calls touches a GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pa():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_pa_build", os.path.join(ROOT, "paged_kv_cache_465_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import paged_kv_cache_465_b200 as pa
    return pa


def _declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\([^;]*\)\s*;", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while", "return")))


def test_exports_every_declared_symbol(pa):
    names = _declared_functions()
    assert "paged_attn_decode" in names and "pa_alloc_append" in names
    lib = ctypes.CDLL(pa.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert pa.version().startswith("pagedattn")


def _state(a):
    return a.free_queue(), [a.ref_count(b) for b in range(a.num_blocks)]


def test_allocator_matches_oracle_random_traces(pa):
    from oracle.paged import RefAllocator, NoBlocks as RefNoBlocks, InvalidCall
    rng = np.random.default_rng(123)
    for trial in range(30):
        nb = int(rng.integers(4, 300))
        order = rng.permutation(nb) if trial % 2 else None
        ref = RefAllocator(nb, 16, order=order)
        nat = pa.BlockAllocator(nb, 16, order=order)
        live, nxt = [], 0
        for step in range(400):
            op = int(rng.integers(0, 5))
            args = None
            if op == 0 or not live:
                args = ("add_seq", nxt, int(rng.integers(0, 120)))
            elif op == 1:
                args = ("fork", live[int(rng.integers(len(live)))], nxt)
            elif op == 2:
                args = ("append", live[int(rng.integers(len(live)))], int(rng.integers(0, 50)))
            elif op == 3:
                # a batch over a random subset (forks share last blocks); now and then a
                # duplicate or unknown id, which both sides must refuse
                k = int(rng.integers(1, len(live) + 1))
                ids = [live[i] for i in rng.choice(len(live), size=k, replace=False)]
                if rng.random() < 0.1:
                    ids.append(ids[0] if rng.random() < 0.5 else nxt + 1000)
                args = ("append_batch", ids, rng.integers(0, 20, len(ids)).tolist())
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
            assert r_exc == n_exc, (args, r_exc, n_exc)
            if r_exc is None:
                if args[0] in ("add_seq", "fork"):
                    live.append(args[1] if args[0] == "add_seq" else args[2])
                    nxt += 1
                if args[0] == "free_seq":
                    live.remove(args[1])
                if args[0] == "add_seq":
                    assert np.array_equal(r_res, n_res)
                if args[0] == "append":
                    assert np.array_equal(r_res[0], n_res[0]) and list(r_res[1]) == n_res[1]
                if args[0] == "append_batch":
                    assert np.array_equal(r_res[0], n_res[0])
                    assert [tuple(p) for p in n_res[1].tolist()] == list(r_res[1])
            assert _state(nat) == (list(ref.free), ref.refs)
            for s in live:
                assert nat.block_table(s) == ref.block_table(s)
                assert nat.seq_len(s) == ref.seq_len(s)


def test_append_batch_equals_single_appends_and_is_atomic(pa):
    """A decode step of 100 forks that share a partial last block: one batch call gives the
    slots, pairs and state of 100 single calls; a batch one block short changes nothing."""
    one, bat = pa.BlockAllocator(256, 16), pa.BlockAllocator(256, 16)
    for a in (one, bat):
        a.add_seq(0, 200)
        for c in range(1, 100):
            a.fork(0, c)
    ids = list(range(99, -1, -1))
    s1, p1 = [], []
    for s in ids:
        sl, pr = one.append(s, 1)
        s1.append(sl)
        p1 += pr
    s2, p2 = bat.append_batch(ids, 1)
    assert np.array_equal(np.concatenate(s1), s2) and p1 == [tuple(p) for p in p2.tolist()]
    assert len(p1) == 99 and _state(one) == _state(bat)
    assert all(one.block_table(s) == bat.block_table(s) for s in ids)
    before = (_state(bat), [bat.block_table(s) for s in ids], [bat.seq_len(s) for s in ids])
    assert bat.num_free() == 256 - 13 - 99
    with pytest.raises(pa.NoBlocks):          # 201 -> 233 tokens: 2 new blocks each, 200 > 144
        bat.append_batch(ids, 32)
    assert before == (_state(bat), [bat.block_table(s) for s in ids], [bat.seq_len(s) for s in ids])
    with pytest.raises(pa.PagedAttnError):
        bat.append_batch([1, 1], 1)


def test_allocator_shared_prefix_example(pa):
    a = pa.BlockAllocator(512, 16)
    a.add_seq(0, 200)
    for c in range(1, 100):
        a.fork(0, c)
    prefix = a.block_table(0)
    pairs = []
    for s in range(100):
        pairs += a.append(s, 50)[1]
    assert len(pairs) == 99 and all(p[0] == prefix[-1] for p in pairs)
    assert [a.ref_count(b) for b in prefix[:12]] == [100] * 12
    assert a.ref_count(prefix[-1]) == 1
    assert 512 - a.num_free() == 412


def test_allocator_rejects_and_stays_unchanged(pa):
    a = pa.BlockAllocator(4, 16)
    a.add_seq(0, 40)
    before = _state(a)
    with pytest.raises(pa.NoBlocks):
        a.add_seq(1, 17)
    with pytest.raises(pa.NoBlocks):
        a.append(0, 30)
    with pytest.raises(pa.PagedAttnError):
        a.add_seq(0, 1)
    with pytest.raises(pa.PagedAttnError):
        a.fork(7, 8)
    assert _state(a) == before
    with pytest.raises(ValueError):
        pa.BlockAllocator(3, 16, order=[0, 0, 1])


def test_host_validation_without_device(pa):
    lib = pa._lib
    d = pa.make_desc(4, 4, 2, 64, 3, 32, 0, pa.PA_F32, pa.PA_F32, pa.PA_F32)
    assert pa.workspace_size(d, 40) == 0
    d2 = pa.make_desc(4, 4, 2, 64, 3, 32, 16, pa.PA_F32, pa.PA_F32, pa.PA_F32)
    assert pa.workspace_size(d2, 40) > 0
    nul = ctypes.c_void_p(0)
    bad = [
        pa.make_desc(4, 5, 2, 64, 3, 32, 0, pa.PA_F32, pa.PA_F32, pa.PA_F32),   # Hq % Hkv
        pa.make_desc(4, 4, 2, 64, 3, 32, 8, pa.PA_F32, pa.PA_F32, pa.PA_F32),   # partition % 16
        pa.make_desc(-1, 4, 2, 64, 3, 32, 0, pa.PA_F32, pa.PA_F32, pa.PA_F32),
    ]
    for b in bad:
        st = lib.paged_attn_decode(nul, nul, nul, nul, nul, ctypes.c_float(0.1), nul,
                                   ctypes.byref(b), 40, nul, nul, nul, nul, nul, nul, 0, nul)
        assert st == pa.PA_ERR_INVALID
    uns = pa.make_desc(4, 4, 2, 96, 3, 32, 0, pa.PA_F32, pa.PA_F32, pa.PA_F32)    # head_dim 96
    st = lib.paged_attn_decode(nul, nul, nul, nul, nul, ctypes.c_float(0.1), nul,
                               ctypes.byref(uns), 40, nul, nul, nul, nul, nul, nul, 0, nul)
    assert st == pa.PA_ERR_UNSUPPORTED
    mixed = pa.make_desc(4, 4, 2, 64, 3, 32, 0, pa.PA_F32, pa.PA_BF16, pa.PA_F32)
    st = lib.paged_attn_decode(nul, nul, nul, nul, nul, ctypes.c_float(0.1), nul,
                               ctypes.byref(mixed), 40, nul, nul, nul, nul, nul, nul, 0, nul)
    assert st == pa.PA_ERR_UNSUPPORTED
    # null pointers with a valid descriptor are rejected before any launch
    st = lib.paged_attn_decode(nul, nul, nul, nul, nul, ctypes.c_float(0.1), nul,
                               ctypes.byref(d), 40, nul, nul, nul, nul, nul, nul, 0, nul)
    assert st == pa.PA_ERR_INVALID
    # split path without workspace
    st = lib.paged_attn_decode(ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256),
                               ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_float(0.1),
                               ctypes.c_void_p(256), ctypes.byref(d2), 40, nul, nul, nul, nul,
                               nul, nul, 0, nul)
    assert st == pa.PA_ERR_WORKSPACE
    # zero-sized work is a successful no-op
    assert lib.reshape_and_cache(nul, nul, nul, nul, nul, 0, 128, 128, 2, 64, 16, 32,
                                 pa.PA_F32, pa.PA_F32, nul, nul, nul, nul, nul) == pa.PA_OK
    assert lib.copy_blocks(nul, nul, nul, nul, nul, nul, nul, 0, 2, 64, 16, 32, pa.PA_BF16,
                           nul) == pa.PA_OK
    assert lib.reshape_and_cache(nul, nul, nul, nul, nul, 3, 128, 128, 2, 60, 16, 32,
                                 pa.PA_F32, pa.PA_F32, nul, nul, nul, nul, nul) == pa.PA_ERR_INVALID
    assert lib.reshape_and_cache(nul, nul, nul, nul, nul, 3, 128, 128, 2, 64, 16, 32,
                                 pa.PA_BF16, pa.PA_F32, nul, nul, nul, nul,
                                 nul) == pa.PA_ERR_UNSUPPORTED
    # int8 caches need scales and zero points
    one = ctypes.c_void_p(256)
    assert lib.reshape_and_cache(one, one, one, one, one, 3, 128, 128, 2, 64, 16, 32,
                                 pa.PA_BF16, pa.PA_INT8, one, one, nul, nul,
                                 nul) == pa.PA_ERR_INVALID
    i8 = pa.make_desc(4, 4, 2, 128, 3, 32, 0, pa.PA_BF16, pa.PA_INT8, pa.PA_BF16)
    st = lib.paged_attn_decode(one, one, one, one, one, ctypes.c_float(0.1), one, ctypes.byref(i8),
                               40, one, one, nul, nul, nul, nul, 0, nul)
    assert st == pa.PA_ERR_INVALID
    assert lib.pa_set_decode_impl(6) == pa.PA_ERR_INVALID
    assert lib.pa_set_decode_impl(-1) == pa.PA_ERR_INVALID
    assert lib.pa_set_decode_impl(0) == pa.PA_OK


def test_binding_refuses_host_tensors(pa):
    import torch
    q = torch.zeros(4, 4, 64)
    kc = torch.zeros(32, 2, 16, 64)
    with pytest.raises(ValueError):
        pa.paged_attn_decode(q, kc, kc, torch.zeros(4, 3, dtype=torch.int32),
                             torch.zeros(4, dtype=torch.int32), 0.125, q.clone(), max_context_len=40)


def test_prefill_host_validation_without_device(pa):
    lib = pa._lib
    nul = ctypes.c_void_p(0)
    one = ctypes.c_void_p(256)
    d = pa.make_desc(4, 32, 8, 128, 64, 1024, 0, pa.PA_BF16, pa.PA_BF16, pa.PA_BF16)

    def call(desc, tokens=100, max_q=50, max_ctx=1024, ptr=one, qs=one, scale=0.1):
        return lib.paged_attn_prefill(ptr, ptr, ptr, ptr, ptr, qs, tokens, max_q,
                                      ctypes.c_float(scale), ptr, ctypes.byref(desc), max_ctx,
                                      nul, nul, nul, nul, nul, nul)
    split = pa.make_desc(4, 32, 8, 128, 64, 1024, 512, pa.PA_BF16, pa.PA_BF16, pa.PA_BF16)
    assert call(split) == pa.PA_ERR_INVALID                     # no split-KV for prefill
    assert call(d, tokens=-1) == pa.PA_ERR_INVALID
    assert call(d, max_q=2000, max_ctx=1024) == pa.PA_ERR_INVALID  # a query past its context
    assert call(d, max_ctx=1025) == pa.PA_ERR_INVALID            # table shorter than context
    assert call(d, scale=float("nan")) == pa.PA_ERR_INVALID
    assert call(d, qs=nul) == pa.PA_ERR_INVALID                  # query_start is required
    assert call(d, tokens=0, ptr=nul, qs=nul) == pa.PA_OK         # nothing to do
    uns = pa.make_desc(4, 32, 8, 96, 64, 1024, 0, pa.PA_BF16, pa.PA_BF16, pa.PA_BF16)
    assert call(uns) == pa.PA_ERR_UNSUPPORTED
    fp8 = pa.make_desc(4, 32, 8, 128, 64, 1024, 0, pa.PA_BF16, pa.PA_FP8_E4M3, pa.PA_BF16)
    assert call(fp8) == pa.PA_ERR_INVALID                        # fp8 needs its scales


def test_library_chosen_partition(pa):
    """PA_PARTITION_AUTO: one pass when no context exceeds 512 tokens, else 512-token
    partitions for at least 1024 (sequence, kv head) pairs and 1024-token ones for fewer;
    the workspace and the launch count follow the chosen partition."""
    for S, Hkv, L, B in [(32, 8, 4096, 16), (256, 8, 8192, 16), (100, 8, 250, 16),
                         (8, 8, 131072, 16), (1, 1, 512, 16), (1, 1, 513, 8), (3, 2, 40, 32),
                         (4096, 8, 600, 32), (64, 8, 1000, 8), (128, 8, 1000, 16),
                         (127, 8, 1000, 16)]:
        d = pa.make_desc(S, 4 * Hkv, Hkv, 128, -(-L // B), 1 << 16, pa.PARTITION_AUTO, pa.PA_BF16,
                         pa.PA_BF16, pa.PA_BF16, block_size=B)
        p = pa.partition_size_for(d, L)
        assert p == (0 if L <= 512 else 512 if S * Hkv >= 1024 else 1024), (S, Hkv, L, p)
        e = pa.make_desc(S, 4 * Hkv, Hkv, 128, -(-L // B), 1 << 16, p, pa.PA_BF16, pa.PA_BF16,
                         pa.PA_BF16, block_size=B)
        assert pa.workspace_size(d, L) == pa.workspace_size(e, L)
        assert pa.decode_launches(d, L) == pa.decode_launches(e, L) > 0
    # an explicit partition is reported as given; a bad one is refused
    d = pa.make_desc(4, 8, 2, 128, 4, 64, 48, pa.PA_BF16, pa.PA_BF16, pa.PA_BF16)
    assert pa.partition_size_for(d, 60) == 48
    d = pa.make_desc(4, 8, 2, 128, 4, 64, -2, pa.PA_BF16, pa.PA_BF16, pa.PA_BF16)
    assert pa.partition_size_for(d, 60) == -1 and pa.workspace_size(d, 60) == 0
