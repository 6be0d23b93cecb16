"""Pins of the oracle's prefill attention (causal attention of a step's new tokens).

Against: the already pinned decode oracle (one new token per sequence is a decode step);
torch's scaled_dot_product_attention with its own causal mask, in float64 on contiguous
per-token arrays taken from the draw (never through the block table): whole prompts
directly, chunks as the last rows of a whole-context causal pass; textbook Python loops;
and causality (K/V after a token's position never changes its row).
"""
import math

import numpy as np
import pytest
import torch

import workloads
from oracle import attention, flows


def _dec(draw, x):
    if draw.wl.in_dtype == "f32":
        return np.asarray(x, np.float32).astype(np.float64)
    return (np.asarray(x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _sdpa_causal(Q, K, V, scale):
    """Q [Hq, n, d], K/V [Hkv, n, d] float64 -> out [Hq, n, d] and lse [Hq, n]."""
    G = Q.shape[0] // K.shape[0]
    Kx = torch.from_numpy(K).repeat_interleave(G, dim=0)
    Vx = torch.from_numpy(V).repeat_interleave(G, dim=0)
    Qt = torch.from_numpy(Q)
    out = torch.nn.functional.scaled_dot_product_attention(Qt, Kx, Vx, is_causal=True,
                                                           scale=scale)
    # lse from the library's logsumexp over the causally masked scores
    z = scale * Qt @ Kx.transpose(1, 2)
    n = Q.shape[1]
    z = z.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    return out.numpy(), torch.logsumexp(z, dim=-1).numpy()


def _scale(draw):
    return float(np.float32(1.0 / math.sqrt(draw.wl.head_dim)))


@pytest.mark.parametrize("kv", ["bf16", "fp8", "int8"])
def test_one_new_token_is_a_decode_step(kv):
    wl = workloads.PREFILL_WORKLOADS["chunked"].scaled(num_seqs=4, new=("chunk", 1),
                                                       lens=("fixed", [1, 17, 300, 1000]),
                                                       num_blocks=256, kv_dtype=kv)
    d = workloads.draw_prefill(wl)
    st = flows.build_prefill_state(d)
    o, l = flows.ref_prefill_outputs(d, st)
    od, ld = attention.ref_decode(d.q, st.k_cache, st.v_cache, st.block_tables,
                                  st.context_lens, _scale(d), wl.num_kv_heads, wl.in_dtype,
                                  wl.kv_dtype, st.k_scales, st.v_scales, k_zeros=st.k_zeros,
                                  v_zeros=st.v_zeros)
    assert np.allclose(o, od, rtol=0, atol=1e-12) and np.allclose(l, ld, rtol=0, atol=1e-12)


@pytest.mark.parametrize("B", [16, 8, 32])
def test_whole_prompts_match_library_causal_attention(B):
    wl = workloads.PREFILL_WORKLOADS["prefill"].scaled(num_seqs=3, lens=("fixed", [1, 45, 200]),
                                                       block_size=B, num_blocks=4096 // B)
    d = workloads.draw_prefill(wl)
    st = flows.build_prefill_state(d)
    o, l = flows.ref_prefill_outputs(d, st)
    for s in range(3):
        k, v = d.kv(s)
        r0, r1 = d.query_start[s], d.query_start[s + 1]
        Q = _dec(d, d.q[r0:r1]).transpose(1, 0, 2)
        ref_o, ref_l = _sdpa_causal(Q, _dec(d, k).transpose(1, 0, 2),
                                    _dec(d, v).transpose(1, 0, 2), _scale(d))
        assert np.allclose(o[r0:r1], ref_o.transpose(1, 0, 2), rtol=0, atol=1e-12)
        assert np.allclose(l[r0:r1], ref_l.T, rtol=0, atol=1e-12)


def test_chunks_are_the_last_rows_of_a_whole_context_pass():
    d = workloads.draw_prefill(workloads.PREFILL_WORKLOADS["chunked"].scaled(
        num_seqs=3, lens=("fixed", [600, 513, 1500]), num_blocks=256))
    st = flows.build_prefill_state(d)
    o, l = flows.ref_prefill_outputs(d, st)
    rng = np.random.default_rng(5)
    wl = d.wl
    for s in range(3):
        ctx, n = int(d.context_lens[s]), int(d.query_lens[s])
        r0 = d.query_start[s]
        k, v = d.kv(s)
        # queries of the cached positions are arbitrary: only the last n rows are compared
        q_all = np.concatenate([rng.standard_normal((ctx - n, wl.num_q_heads, wl.head_dim)),
                                _dec(d, d.q[r0:r0 + n])])
        ref_o, ref_l = _sdpa_causal(q_all.transpose(1, 0, 2), _dec(d, k).transpose(1, 0, 2),
                                    _dec(d, v).transpose(1, 0, 2), _scale(d))
        assert np.allclose(o[r0:r0 + n], ref_o[:, ctx - n:].transpose(1, 0, 2), rtol=0,
                           atol=1e-12)
        assert np.allclose(l[r0:r0 + n], ref_l[:, ctx - n:].T, rtol=0, atol=1e-12)


def test_tiny_against_textbook_loops():
    d = workloads.draw_prefill("prefill_tiny")
    st = flows.build_prefill_state(d)
    o, l = flows.ref_prefill_outputs(d, st)
    wl = d.wl
    for s in range(wl.num_seqs):
        k, v = d.kv(s)
        K, V = _dec(d, k), _dec(d, v)
        ctx, n = int(d.context_lens[s]), int(d.query_lens[s])
        for i in range(n):
            p = ctx - n + i
            row = d.query_start[s] + i
            for h in range(wl.num_q_heads):
                kvh = h // wl.group
                ref, lse = attention.brute_force_attention(
                    _dec(d, d.q[row, h]), K[:p + 1, kvh].tolist(), V[:p + 1, kvh].tolist(),
                    _scale(d))
                assert np.allclose(o[row, h], ref, rtol=0, atol=1e-12)
                assert l[row, h] == pytest.approx(lse, abs=1e-12)


def test_later_positions_never_change_a_row():
    d = workloads.draw_prefill("prefill_tiny")
    st = flows.build_prefill_state(d)
    o1, l1 = flows.ref_prefill_outputs(d, st)
    # sequence 2: context 40, new tokens at positions 24..39; overwrite position 39's K/V
    s, p = 2, 39
    blk = st.block_tables[s][p // d.wl.block_size]
    off = p % d.wl.block_size
    st.k_cache[blk, :, off] += 3.0
    st.v_cache[blk, :, off] -= 5.0
    o2, l2 = flows.ref_prefill_outputs(d, st)
    r_last = d.query_start[s + 1] - 1
    assert np.array_equal(o1[:r_last], o2[:r_last]) and np.array_equal(l1[:r_last], l2[:r_last])
    assert not np.allclose(o1[r_last], o2[r_last])
