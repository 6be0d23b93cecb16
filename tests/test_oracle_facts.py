"""Pins of the closed-form sizes against the numbers the pages print (tests/golden/)."""
import math

import numpy as np
import pytest

from oracle import facts


def test_kv_bytes_worked_example(golden):
    g = golden("kv_size_example.json")
    a = g["assumptions"]
    per_tok = facts.kv_cache_bytes(a["num_layers"], a["num_kv_heads"], a["head_dim"],
                                   a["dtype_bytes"], tokens=1)
    assert per_tok == g["bytes_per_token_per_request"] == 131072
    per_req = facts.kv_cache_bytes(a["num_layers"], a["num_kv_heads"], a["head_dim"],
                                   a["dtype_bytes"], tokens=g["tokens_per_request"])
    assert per_req == g["bytes_per_request"] == 512 * 2 ** 20
    allr = facts.kv_cache_bytes(a["num_layers"], a["num_kv_heads"], a["head_dim"],
                                a["dtype_bytes"], tokens=g["tokens_per_request"],
                                batch=g["concurrent_requests"])
    assert allr == g["bytes_all_requests"] == 16 * 2 ** 30


def test_kv_bytes_linear_in_every_factor():
    base = facts.kv_cache_bytes(3, 5, 7, 2, 11, batch=13)
    assert facts.kv_cache_bytes(6, 5, 7, 2, 11, batch=13) == 2 * base
    assert facts.kv_cache_bytes(3, 10, 7, 2, 11, batch=13) == 2 * base
    assert facts.kv_cache_bytes(3, 5, 14, 2, 11, batch=13) == 2 * base
    assert facts.kv_cache_bytes(3, 5, 7, 1, 11, batch=13) * 2 == base   # fp8 halves fp16
    assert facts.kv_cache_bytes(3, 5, 7, 2, 22, batch=13) == 2 * base
    assert base == 2 * 3 * 5 * 7 * 2 * 11 * 13


def test_gqa_ratios(golden):
    g = golden("gqa_ratio.json")
    mha = facts.kv_cache_bytes(32, g["num_q_heads"], 128, 2, 1)
    for c in g["cases"]:
        r = 100.0 * facts.kv_cache_bytes(32, c["num_kv_heads"], 128, 2, 1) / mha
        assert round(r) == c["printed_percent"]   # 100, 25, 3.125 ~ "about 3 %"


def test_block_table_example(golden):
    g = golden("block_table_example.json")
    for r in g["requests"]:
        assert facts.blocks_for_tokens(r["tokens"], g["block_size"]) == r["blocks"]
        assert facts.last_block_fill(r["tokens"], g["block_size"]) == r["fills"][-1]
        assert sum(r["fills"]) == r["tokens"]


def test_fragmentation_theorem(golden):
    g = golden("fragmentation_bound.json")
    B, T = g["block_size"], g["T"]
    assert 100 * facts.waste_bound(T, B) == pytest.approx(0.78125)
    assert 100 * facts.waste_bound(T, B) > g["waste_bound_printed_percent_below"] - 0.01
    rng = np.random.default_rng(0)
    for _ in range(200):
        lens = rng.integers(T, 4 * T, size=rng.integers(1, 64)).tolist()
        w = facts.paged_waste_fraction(lens, B)
        assert w < facts.waste_bound(T, B)
        for t in lens:
            slack = facts.blocks_for_tokens(t, B) * B - t
            assert 0 <= slack <= g["last_block_slack_max_tokens"]
    # worst case: every request one token past a block boundary
    worst = [T + 1] * 10
    assert facts.paged_waste_fraction(worst, B) == pytest.approx(15 / (T + 16))
    c = g["contiguous_internal_fragmentation"]
    assert 100 * facts.internal_fragmentation_contiguous(c["T"], c["T_max"]) == c["printed_percent"]


def test_sharing_savings(golden):
    g = golden("prefix_sharing.json")
    assert 100 * facts.sharing_savings_prefix_only(g["prefix_only"]["R"]) == pytest.approx(99.0)
    p = g["prefix_and_suffix"]
    s = facts.sharing_savings(p["R"], p["p"], p["s_bar"])
    assert round(100 * s, 1) == p["printed_percent"]
    assert s == pytest.approx(0.792)
    o = g["block_table_overhead"]
    # int32 entries, a 2048-token longest context, 16-token blocks (a reading)
    b = facts.block_table_bytes(o["requests"], 2048)
    assert b == 131072
    assert abs(b - o["printed_bytes_approx"]) / o["printed_bytes_approx"] < 0.01


@pytest.mark.parametrize("B", [8, 32])
def test_fragmentation_bound_other_block_sizes(B):
    """[Ch4PA] Theorem 1 trade-off note: halving the block size halves the bound, doubling
    doubles it; the proof's step (at most B - 1 idle slots per request) holds for any B."""
    T = 2048
    assert facts.waste_bound(T, B) == facts.waste_bound(T, 16) * B / 16
    rng = np.random.default_rng(B)
    for _ in range(200):
        lens = rng.integers(T, 4 * T, size=rng.integers(1, 64)).tolist()
        assert facts.paged_waste_fraction(lens, B) < facts.waste_bound(T, B)
        for t in lens:
            assert 0 <= facts.blocks_for_tokens(t, B) * B - t <= B - 1
    # every request one token past a boundary: B - 1 idle slots each
    assert facts.paged_waste_fraction([T + 1] * 7, B) == pytest.approx((B - 1) / (T + B))
