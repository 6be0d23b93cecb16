"""GPU parity of prefill attention (paged_attn_prefill) against the oracle.

Within the per-dtype tolerances of tests/gpu_common.py: whole prompts, chunks after cached
tokens, one-token steps, mixed batches with sequences that bring nothing, every group size
and block size of the tensor-core kernel, the CUDA-core path for the other dtypes and
shapes. Cache contents after the step's writes are bit-exact. Bit-identical: rows before a
changed key (causality) and outputs under a different physical placement.
"""
import numpy as np
import pytest

import workloads
from oracle import flows
from tests.gpu_common import compare_decode, cache_codes

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_465_b200 as pa
    pa.set_decode_impl("auto")
    yield pa
    pa.set_decode_impl("auto")


@pytest.fixture(scope="module")
def scen():
    from paged_kv_cache_465_b200.scenario import PrefillScenario
    return PrefillScenario


def _run(pa, scen, draw, impl="auto", draw_seqs=None, check_cache=True):
    pa.set_decode_impl(impl)
    try:
        sc = scen(draw, draw_seqs=draw_seqs)
        sc.step()
        torch.cuda.synchronize()
        assert pa.device_error() == 0
        st = flows.build_prefill_state(draw, write_seqs=draw_seqs)
        seqs = sorted(sc.draw_seqs)
        out_ref, lse_ref = flows.ref_prefill_outputs(draw, st, seqs=seqs)
        rows = np.concatenate([np.arange(draw.query_start[s], draw.query_start[s + 1])
                               for s in seqs]).astype(np.int64)
        stats = compare_decode(sc.out, sc.lse, out_ref, lse_ref, draw.wl.kv_dtype, seqs=rows)
        if check_cache:
            assert np.array_equal(sc.block_tables.cpu().numpy(), st.block_tables)
            assert np.array_equal(cache_codes(sc.cache.k_cache), st.k_cache)
            assert np.array_equal(cache_codes(sc.cache.v_cache), st.v_cache)
        return sc, stats
    finally:
        pa.set_decode_impl("auto")


IMPLS = ["simt", "auto"]   # "auto": the tensor-core kernel where the shape allows it


@pytest.mark.parametrize("impl", IMPLS)
def test_tiny_fp32(pa, scen, impl):
    _run(pa, scen, workloads.draw_prefill("prefill_tiny"), impl)


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("lens,new", [
    ([1, 45, 700], ("full",)),                       # whole prompts
    ([600, 513, 1500, 2000], ("chunk", 512)),        # chunks after cached tokens
    ([1, 130, 129, 4000], ("chunk", 1)),             # one new token: a decode step
    ([300, 17, 5, 1000, 64], ("uniform", 0, 300)),   # ragged, some sequences bring nothing
])
def test_bf16_shapes(pa, scen, impl, lens, new):
    wl = workloads.PREFILL_WORKLOADS["chunked"].scaled(num_seqs=len(lens), lens=("fixed", lens),
                                                       new=new, num_blocks=1024)
    _run(pa, scen, workloads.draw_prefill(wl), impl)


@pytest.mark.parametrize("B", [8, 32])
@pytest.mark.parametrize("impl", IMPLS)
def test_block_sizes(pa, scen, B, impl):
    wl = workloads.PREFILL_WORKLOADS["chunked"].scaled(
        num_seqs=4, lens=("fixed", [333, 128, 129, 1100]), new=("chunk", 300),
        block_size=B, num_blocks=16384 // B)
    _run(pa, scen, workloads.draw_prefill(wl), impl)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (64, 8), (16, 1), (12, 2)])
def test_group_sizes(pa, scen, hq, hkv):
    wl = workloads.PREFILL_WORKLOADS["chunked"].scaled(
        num_seqs=3, num_q_heads=hq, num_kv_heads=hkv, lens=("fixed", [200, 77, 900]),
        new=("chunk", 160), num_blocks=512)
    _run(pa, scen, workloads.draw_prefill(wl))


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("kv", ["fp8", "int8"])
@pytest.mark.parametrize("B", [8, 16, 32])
def test_quantised_caches(pa, scen, impl, kv, B):
    """fp8 / int8 caches: the tensor-core kernel dequantises staged codes to bf16 in shared
    memory (per-block scale and zero point); the CUDA-core kernel reads them directly."""
    wl = workloads.PREFILL_WORKLOADS["chunked"].scaled(
        num_seqs=4, kv_dtype=kv, block_size=B, num_blocks=16384 // B,
        lens=("fixed", [1, 200, 777, 1500]), new=("chunk", 300))
    _run(pa, scen, workloads.draw_prefill(wl), impl)


@pytest.mark.parametrize("kv,dim", [("fp8", 128), ("int8", 128), ("bf16", 64), ("bf16", 256)])
def test_other_dtypes_and_head_dims(pa, scen, kv, dim):
    wl = workloads.PREFILL_WORKLOADS["chunked"].scaled(
        num_seqs=3, head_dim=dim, kv_dtype=kv, lens=("fixed", [40, 300, 700]),
        new=("chunk", 100), num_blocks=512)
    _run(pa, scen, workloads.draw_prefill(wl))


def test_full_size_prompts_sampled(pa, scen):
    d = workloads.draw_prefill("prefill")
    _run(pa, scen, d, draw_seqs=[0, 5], check_cache=False)


def test_full_size_chunks_sampled(pa, scen):
    d = workloads.draw_prefill("chunked")
    _run(pa, scen, d, draw_seqs=[int(np.argmax(d.context_lens)), 3], check_cache=False)


def test_full_size_fp8_chunks_sampled(pa, scen):
    """The fp8 chunked step the bench times, at full size, on sampled sequences."""
    d = workloads.draw_prefill("chunked_fp8")
    _run(pa, scen, d, draw_seqs=[int(np.argmax(d.context_lens)), int(np.argmin(d.context_lens))],
         check_cache=False)


@pytest.mark.parametrize("impl", IMPLS)
def test_causality_and_placement(pa, scen, impl):
    wl = workloads.PREFILL_WORKLOADS["chunked"].scaled(num_seqs=3, lens=("fixed", [700, 260, 900]),
                                                       new=("chunk", 260), num_blocks=512)
    pa.set_decode_impl(impl)
    try:
        d = workloads.draw_prefill(wl)
        s1 = scen(d)
        s1.step()
        o1 = s1.out.clone()
        # a different physical placement of the same logical KV
        d2 = workloads.draw_prefill(wl)
        d2.pool_order = np.roll(d2.pool_order[::-1], 3).copy()
        s2 = scen(d2)
        s2.step()
        torch.cuda.synchronize()
        assert not torch.equal(s1.block_tables, s2.block_tables)
        assert torch.equal(o1, s2.out) and torch.equal(s1.lse, s2.lse)
        # change the last key of sequence 2: only its last row may change
        s1.step_k[-1] += 4.0
        s1.step()
        torch.cuda.synchronize()
        r_last = int(d.query_start[3]) - 1
        assert torch.equal(o1[:r_last], s1.out[:r_last])
        assert not torch.equal(o1[r_last], s1.out[r_last])
    finally:
        pa.set_decode_impl("auto")


@pytest.mark.parametrize("impl", IMPLS)
def test_error_flags(pa, impl):
    S, Hq, Hkv, d, B, NB = 2, 32, 8, 128, 16, 64
    kc = torch.randn(NB, Hkv, B, d, device="cuda").to(torch.bfloat16)
    vc = torch.randn(NB, Hkv, B, d, device="cuda").to(torch.bfloat16)
    q = torch.randn(40, Hq, d, device="cuda").to(torch.bfloat16)
    out = torch.zeros_like(q)
    bt = torch.tensor([[0, 1, 2, 3], [4, 5, 6, 7]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([30, 40], dtype=torch.int32, device="cuda")
    pa.set_decode_impl(impl)
    try:
        assert pa.device_error() == 0
        # sequence 0 claims more new tokens than its context: skipped and flagged
        qs = torch.tensor([0, 35, 40], dtype=torch.int32, device="cuda")
        pa.paged_attn_prefill(q, kc, vc, bt, lens, qs, 0.1, out, max_query_len=40,
                              max_context_len=64)
        assert pa.device_error() & pa.PA_DEVERR_QUERY
        assert pa.device_error() == 0
        # an out-of-range block id is skipped and flagged; outputs stay finite
        bad = torch.tensor([[0, 1_000_000, 2, 3], [4, 5, 6, 7]], dtype=torch.int32,
                           device="cuda")
        qs = torch.tensor([0, 20, 40], dtype=torch.int32, device="cuda")
        pa.paged_attn_prefill(q, kc, vc, bad, lens, qs, 0.1, out, max_query_len=20,
                              max_context_len=64)
        assert pa.device_error() & pa.PA_DEVERR_BLOCK_ID
        assert pa.device_error() == 0
        assert torch.isfinite(out.float()).all()
    finally:
        pa.set_decode_impl("auto")
