"""Pins of the oracle's decode attention.

Against: textbook attention written as Python loops over contiguous per-token arrays
(never through a block table), closed forms (one token; zero query; identical keys),
SciPy's logsumexp, invariance under the physical placement of blocks, shared-prefix
sequences matching private unshared copies, and one-byte caches against float attention on
values decoded independently (torch's E4M3 decoder; code minus zero point).
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import workloads
from oracle import attention, flows, paged


def _contig(draw, s):
    k, v = draw.kv(s)
    dec = (lambda x: x.astype(np.float64)) if draw.wl.in_dtype == "f32" else \
        (lambda x: (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    return dec(k), dec(v), dec(draw.q[s])


@pytest.mark.parametrize("B,nb", [(16, 32), (8, 64), (32, 16)])
def test_tiny_against_textbook_loops(B, nb):
    d = workloads.draw(workloads.WORKLOADS["tiny"].scaled(block_size=B, num_blocks=nb))
    st = flows.build_state(d)
    out, lse = flows.ref_outputs(d, st)
    wl = d.wl
    for s in range(wl.num_seqs):
        K, V, Q = _contig(d, s)
        for h in range(wl.num_q_heads):
            kvh = h // wl.group
            o, l = attention.brute_force_attention(Q[h], K[:, kvh].tolist(), V[:, kvh].tolist(),
                                                   1.0 / math.sqrt(wl.head_dim))
            assert np.allclose(out[s, h], o, rtol=0, atol=1e-12)
            assert lse[s, h] == pytest.approx(l, abs=1e-12)


@pytest.mark.parametrize("B", [16, 8, 32])
def test_lse_matches_scipy(B):
    d = workloads.draw(workloads.WORKLOADS["b32"].scaled(num_seqs=3, num_blocks=16384 // B,
                                                        block_size=B),
                       lens_override=[7, 300, 1000])
    st = flows.build_state(d)
    out, lse = flows.ref_outputs(d, st)
    sc = float(np.float32(1 / math.sqrt(128)))
    for s in range(3):
        K, V, Q = _contig(d, s)
        for h in (0, 5, 31):
            z = sc * (K[:, h // 4] @ Q[h])
            assert lse[s, h] == pytest.approx(logsumexp(z), abs=1e-12)
            w = np.exp(z - logsumexp(z))
            assert np.allclose(out[s, h], w @ V[:, h // 4], atol=1e-12)


def test_closed_forms():
    rng = np.random.default_rng(0)
    NB, H, B, dd, G = 8, 2, 16, 16, 3
    kc = paged.new_cache(NB, H, B, dd, "f32")
    vc = paged.new_cache(NB, H, B, dd, "f32")
    kc[:] = rng.standard_normal(kc.shape)
    vc[:] = rng.standard_normal(vc.shape)
    bt = np.array([[5, 2, 7, -1], [1, -1, -1, -1], [3, 0, 4, 6]], np.int32)
    lens = np.array([40, 1, 64], np.int32)
    q = rng.standard_normal((3, H * G, dd)).astype(np.float32)
    out, lse = attention.ref_decode(q, kc, vc, bt, lens, 0.3, H, "f32", "f32")
    # one token: the output is that token's value, lse its logit
    for h in range(H * G):
        assert np.array_equal(out[1, h], vc[1, h // G, 0].astype(np.float64))
        assert lse[1, h] == pytest.approx(0.3 * float(q[1, h] @ kc[1, h // G, 0].astype(np.float64)))
    # zero query: uniform weights, out = mean of V over the context, lse = log(ctx)
    q0 = np.zeros_like(q)
    out0, lse0 = attention.ref_decode(q0, kc, vc, bt, lens, 0.3, H, "f32", "f32")
    for s in range(3):
        K, V = attention.gather_kv(kc, vc, bt[s], lens[s], 1, "f32")
        assert np.allclose(out0[s, G:2 * G], V.mean(axis=0), atol=1e-12)
        assert np.allclose(lse0[s], math.log(lens[s]), atol=1e-12)
    # identical keys: uniform weights whatever the query
    kc2 = kc.copy()
    kc2[:] = kc[0, 0, 0]
    out2, _ = attention.ref_decode(q, kc2, vc, bt, lens, 0.3, H, "f32", "f32")
    assert np.allclose(out2, out0, atol=1e-12)
    # empty context
    out3, lse3 = attention.ref_decode(q, kc, vc, bt, np.array([0, 1, 2], np.int32), 0.3, H,
                                      "f32", "f32")
    assert np.all(out3[0] == 0) and np.all(np.isneginf(lse3[0]))


def test_gqa_head_mapping():
    """Query head h reads kv head h // G: make each kv head's values a constant."""
    NB, H, B, dd, G = 4, 4, 16, 8, 2
    kc = paged.new_cache(NB, H, B, dd, "f32")
    vc = paged.new_cache(NB, H, B, dd, "f32")
    for h in range(H):
        vc[:, h] = 10.0 * h + 1
    kc[:] = np.random.default_rng(1).standard_normal(kc.shape)
    q = np.random.default_rng(2).standard_normal((1, H * G, dd)).astype(np.float32)
    out, _ = attention.ref_decode(q, kc, vc, np.array([[2, 0]], np.int32),
                                  np.array([20], np.int32), 0.5, H, "f32", "f32")
    for h in range(H * G):
        assert np.allclose(out[0, h], 10.0 * (h // G) + 1, atol=1e-12)


@pytest.mark.parametrize("name", ["tiny", "b32"])
def test_invariant_under_physical_placement(name):
    wl = workloads.WORKLOADS[name]
    if name == "b32":
        wl = wl.scaled(num_seqs=5, num_blocks=2048)
    d1 = workloads.draw(wl)
    st1 = flows.build_state(d1)
    d2 = workloads.draw(wl)
    d2.pool_order = np.arange(wl.num_blocks, dtype=np.int32)[::-1].copy()
    st2 = flows.build_state(d2)
    assert not np.array_equal(st1.block_tables, st2.block_tables)
    o1, l1 = flows.ref_outputs(d1, st1)
    o2, l2 = flows.ref_outputs(d2, st2)
    assert np.allclose(o1, o2, atol=1e-12, rtol=0) and np.allclose(l1, l2, atol=1e-12, rtol=0)


def test_shared_prefix_matches_unshared_copies():
    wl = workloads.WORKLOADS["shared"].scaled(num_seqs=10)
    d = workloads.draw(wl)
    sh = flows.build_state(d, shared=True)
    un = flows.build_state(d, shared=False)
    assert len(sh.cow_pairs) == 9 and not un.cow_pairs
    used_sh = sh.alloc.num_blocks - sh.alloc.num_free()
    used_un = un.alloc.num_blocks - un.alloc.num_free()
    assert used_sh == 12 + 10 + 30 and used_un == 160
    o1, l1 = flows.ref_outputs(d, sh)
    o2, l2 = flows.ref_outputs(d, un)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


@pytest.mark.parametrize("B", [16, 8, 32])
def test_fp8_dequant_is_code_times_scale(B):
    wl = workloads.WORKLOADS["b256"].scaled(num_seqs=3, num_blocks=4096 // B, block_size=B)
    d = workloads.draw(wl, lens_override=[16, 33, 500])
    st = flows.build_state(d)
    out, lse = flows.ref_outputs(d, st)
    # the decoded cache stays within one E4M3 rounding step of the bf16 inputs
    for s in range(3):
        k, v = d.kv(s)
        kf = (k.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        K, V = attention.gather_kv(st.k_cache, st.v_cache, st.block_tables[s],
                                   int(d.context_lens[s]), 2, "fp8", st.k_scales, st.v_scales)
        err = np.abs(K - kf[:, 2])
        blk = np.arange(len(K)) // B
        sc = st.k_scales[st.block_tables[s][blk], 2][:, None]
        # relative step of E4M3 is 2^-3 for normals -> half-step error <= 2^-4 |x|,
        # subnormal step 2^-9 * scale
        assert np.all(err <= np.maximum(np.abs(kf[:, 2]) * 2 ** -4, 2 ** -10 * sc) + 1e-12)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))


@pytest.mark.parametrize("kv", ["fp8", "int8"])
def test_quantised_attention_on_dequantised_values(kv):
    """One-byte caches: the attention equals float attention over values decoded on their
    own: fp8 codes through torch's float8_e4m3fn, int8 as (code - zero point); each times
    its block's scale, K and V with separate scales (and zero points), gathered token by
    token in a Python loop."""
    rng = np.random.default_rng(21)
    NB, H, B, dd, G = 24, 2, 16, 32, 3
    if kv == "fp8":
        codes = rng.integers(0, 256, (2, NB, H, B, dd)).astype(np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x38                   # no NaN patterns
        kc, vc = codes
        zk = zv = None
        dec = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    else:
        kc, vc = rng.integers(-128, 128, (2, NB, H, B, dd)).astype(np.int8)
        zk = rng.integers(-30, 31, (NB, H)).astype(np.int32)
        zv = rng.integers(-30, 31, (NB, H)).astype(np.int32)
        dec = np.stack([kc.astype(np.int64) - zk[:, :, None, None],
                        vc.astype(np.int64) - zv[:, :, None, None]]).astype(np.float64)
    ks = rng.uniform(0.002, 0.02, (NB, H)).astype(np.float32)
    vs = rng.uniform(0.5, 3.0, (NB, H)).astype(np.float32)
    lens = np.array([1, 16, 17, 90], np.int32)
    perm = rng.permutation(NB)
    bt = np.full((4, 6), -1, np.int32)
    used = 0
    for s, n in enumerate(lens):
        nb = -(-int(n) // B)
        bt[s, :nb] = perm[used:used + nb]
        used += nb
    q = rng.standard_normal((4, H * G, dd)).astype(np.float32)
    sc = 0.7
    out, lse = attention.ref_decode(q, kc, vc, bt, lens, sc, H, "f32", kv, ks, vs,
                                    k_zeros=zk, v_zeros=zv)
    for s, n in enumerate(lens):
        for h in range(H * G):
            kvh = h // G
            K = np.array([dec[0, bt[s, t // B], kvh, t % B] * float(ks[bt[s, t // B], kvh])
                          for t in range(n)])
            V = np.array([dec[1, bt[s, t // B], kvh, t % B] * float(vs[bt[s, t // B], kvh])
                          for t in range(n)])
            z = sc * (K @ q[s, h].astype(np.float64))
            w = np.exp(z - logsumexp(z))
            assert lse[s, h] == pytest.approx(logsumexp(z), abs=1e-12)
            assert np.allclose(out[s, h], w @ V, rtol=0, atol=1e-12 * np.abs(V).max())
