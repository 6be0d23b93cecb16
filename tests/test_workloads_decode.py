"""The decode input recipe: seeded and reproducible draws with the length distributions the
workloads name (fixed tiny lengths, U{1..4096}, lognormal(ln 1024, 1) clipped to
[16, 8192], 200 shared + 50 private tokens, 131072 each), a permuted block pool, and block
scales that do what the recipe says: fp8 absmax / 448 puts every block's largest value on
E4M3's largest finite magnitude; int8 min / max puts the block's range on the byte's range.
"""
import math

import numpy as np
import pytest

import workloads
from oracle import codecs


def test_draws_are_reproducible():
    for name in ("tiny", "b32", "b256"):
        d1, d2 = workloads.draw(name), workloads.draw(name)
        assert np.array_equal(d1.context_lens, d2.context_lens)
        assert np.array_equal(d1.pool_order, d2.pool_order)
        assert np.array_equal(d1.q, d2.q)
        assert np.array_equal(d1.kv(1)[1], d2.kv(1)[1])
    assert not np.array_equal(workloads.draw("b32").q[:4], workloads.draw("b256").q[:4])


def test_query_scale_option_scales_before_bf16_rounding():
    # the q dynamic-range parity case: per-element factors applied to the float32 draw,
    # then rounded to bf16 like every bf16 input; K/V and lengths are untouched
    wl = workloads.WORKLOADS["b256"].scaled(num_seqs=3)
    base = workloads.draw(wl, lens_override=[5, 40, 700])
    f = np.full((3, wl.num_q_heads, wl.head_dim), 2.0 ** -6, dtype=np.float32)
    f[:, 1::4] = 2.0 ** 3
    d = workloads.draw(wl, lens_override=[5, 40, 700], q_scale=f)
    # power-of-two factors commute with bf16 rounding (no under- or overflow here)
    expect = codecs.bf16_decode(base.q).astype(np.float64) * f
    assert np.array_equal(codecs.bf16_decode(d.q).astype(np.float64), expect)
    assert np.array_equal(d.kv(2)[0], base.kv(2)[0])
    assert np.array_equal(d.context_lens, base.context_lens)


def test_length_distributions():
    W = workloads.WORKLOADS
    assert workloads.draw("tiny").context_lens.tolist() == [5, 16, 17, 40]
    b32 = workloads.draw("b32").context_lens
    assert b32.size == 32 and b32.min() >= 1 and b32.max() <= 4096
    b256 = workloads.draw("b256").context_lens
    assert b256.size == 256 and b256.min() >= 16 and b256.max() <= 8192
    # lognormal(ln 1024, 1): the sample median of 256 draws is within a few standard errors
    # of 1024 (the log-median's standard error is about 1.25 / sqrt(256) = 0.08)
    assert abs(math.log(np.median(b256)) - math.log(1024)) < 0.3
    # a much larger draw of the same recipe: about 2 % clipped at 8192 (P[N(0,1) > ln 8])
    big = workloads.draw(W["b256"].scaled(num_seqs=20000, num_blocks=4096)).context_lens
    assert abs((big == 8192).mean() - 0.5 * math.erfc(math.log(8) / math.sqrt(2))) < 0.005
    assert set(workloads.draw("long").context_lens.tolist()) == {131072}
    sh = workloads.draw("shared")
    assert set(sh.context_lens.tolist()) == {250}
    # the shared prefix is the same 200 tokens in every sequence, the suffixes differ
    k0, k1 = sh.kv(0)[0], sh.kv(1)[0]
    assert np.array_equal(k0[:200], k1[:200]) and not np.array_equal(k0[200:], k1[200:])


def test_pool_is_a_permutation_and_values_are_standard_normal():
    d = workloads.draw("b32")
    assert np.array_equal(np.sort(d.pool_order), np.arange(workloads.WORKLOADS["b32"].num_blocks))
    k, _ = d.kv(3)
    x = codecs.bf16_decode(k).ravel()
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1.0) < 0.02


@pytest.mark.parametrize("s", [0, 7, 100])
def test_fp8_scales_put_the_block_absmax_on_448(s):
    d = workloads.draw("b256")
    B = d.wl.block_size
    k, v = d.kv(s)
    ks, vs = d.fp8_scales_logical(s)
    n = int(d.context_lens[s])
    for x, sc in ((k, ks), (v, vs)):
        xf = codecs.bf16_decode(x)
        for b in range(-(-n // B)):
            blk = np.abs(xf[b * B:(b + 1) * B])            # [tokens, Hkv, d]
            y = blk.max(axis=(0, 2)) / sc[b].astype(np.float64)
            assert np.allclose(y, 448.0, rtol=2e-7)
            codes = codecs.e4m3_encode((blk / sc[b][None, :, None]).astype(np.float32))
            assert np.all((codes & 0x7F) <= 0x7E)            # nothing saturates past 448


@pytest.mark.parametrize("s", [0, 9])
def test_int8_params_put_the_block_range_on_the_byte_range(s):
    wl = workloads.WORKLOADS["b256_int8"].scaled(num_seqs=12)
    d = workloads.draw(wl)
    B = wl.block_size
    k, _ = d.kv(s)
    ks, kz, _, _ = d.int8_params_logical(s)
    n = int(d.context_lens[s])
    xf = codecs.bf16_decode(k).astype(np.float32)
    for b in range(-(-n // B)):
        blk = xf[b * B:min(n, (b + 1) * B)]
        for h in range(wl.num_kv_heads):
            c = codecs.int8_encode((blk[:, h] / ks[b, h]).astype(np.float32), kz[b, h])
            # the block's minimum lands on -128 (or one code above, by rounding) and its
            # maximum on 127 (or one below); nothing outside is clipped by more than a step
            assert c.min() <= -127 and c.max() >= 126
            back = (c.astype(np.float64) - kz[b, h]) * ks[b, h]
            assert np.max(np.abs(back - blk[:, h])) <= ks[b, h] * 1.0 + 1e-6


@pytest.mark.parametrize("name", ["tiny", "b32", "shared"])
def test_decode_state_layout(name):
    """The oracle's state builder against the draw, token by token: every cached token's K
    and V sit at slot table[t // B] * B + t % B with the draw's values (bf16 / f32 bits
    unchanged), the step token is the last position, tables use ceil(ctx / B) blocks, and
    sequences share physical blocks only on the shared-prefix workload."""
    from oracle import flows
    wl = workloads.WORKLOADS[name]
    if name == "b32":
        wl = wl.scaled(num_seqs=6, num_blocks=1024)
    d = workloads.draw(wl)
    st = flows.build_state(d)
    B = wl.block_size
    owners = {}
    for s in range(wl.num_seqs):
        n = int(d.context_lens[s])
        row = st.block_tables[s]
        nblk = -(-n // B)
        assert np.all(row[:nblk] >= 0) and np.all(row[nblk:] == -1)
        for b in row[:nblk]:
            owners.setdefault(int(b), set()).add(s)
        k, v = d.kv(s)
        t = np.arange(n)
        blk, off = row[t // B], t % B
        assert np.array_equal(st.k_cache[blk, :, off, :], k)
        assert np.array_equal(st.v_cache[blk, :, off, :], v)
        last = n - 1
        assert st.step_slots[s].tolist()[-1] == int(row[last // B]) * B + last % B
    shared = [b for b, o in owners.items() if len(o) > 1]
    if name == "shared":
        # the 12 full blocks of the 200-token prefix are shared by all 100 sequences; the
        # partial 13th was copied on write by 99 of them
        assert len(shared) == 12 and all(len(owners[b]) == 100 for b in shared)
        assert len(st.cow_pairs) == 99
    else:
        assert not shared and not st.cow_pairs
