"""The allocation-free decode entry point, through the C ABI.

Some callers cannot allocate device memory (code running under stream capture, plugins in
a host runtime that owns all device allocations, callers with no workspace to pass). For
them the library serves the split-KV scratch from a fixed array of its own. This checks,
on two calls in a row with different shapes and dtypes (the second call finds the first
call's leftovers in the shared array), that its results match the workspace entry point
within the parity tolerances, and that a request larger than the array is refused.
"""
import ctypes

import pytest

import workloads

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _call_noalloc(pa, sc, out, lse):
    desc = pa.decode_desc_for(sc.q, sc.cache.k_cache, sc.block_tables, sc.partition_size)
    c = sc.cache
    st = pa._lib.paged_attn_decode_noalloc(
        _ptr(sc.q), _ptr(c.k_cache), _ptr(c.v_cache), _ptr(sc.block_tables),
        _ptr(sc.context_lens), ctypes.c_float(sc.scale), _ptr(out), ctypes.byref(desc),
        int(sc.max_context_len), _ptr(c.k_scales), _ptr(c.v_scales), _ptr(c.k_zeros),
        _ptr(c.v_zeros), _ptr(lse),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, desc


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_465_b200 as pa
    from paged_kv_cache_465_b200.scenario import DeviceScenario
    from tests.gpu_common import TOL
    pa.set_decode_impl("auto")
    cases = [
        (workloads.WORKLOADS["b256"].scaled(num_seqs=24), None, 512),
        (workloads.WORKLOADS["long"].scaled(num_seqs=3), [9000, 700, 2500], 512),
    ]
    for wl, lens, part in cases:
        draw = workloads.draw(wl, lens_override=lens)
        sc = DeviceScenario(draw, draw_seqs=[], partition_size=part)
        sc.step()  # cache write + decode through the workspace entry point
        torch.cuda.synchronize()
        ref_out, ref_lse = sc.out.clone(), sc.lse.clone()
        out = torch.full_like(sc.out, float("nan"))
        lse = torch.full_like(sc.lse, float("nan"))
        st, desc = _call_noalloc(pa, sc, out, lse)
        assert st == pa.PA_OK
        torch.cuda.synchronize()
        assert pa.device_error() == 0
        assert pa.workspace_size(desc, sc.max_context_len) > 0
        tol = TOL[wl.kv_dtype]
        assert float((out.float() - ref_out.float()).abs().max()) <= tol["max_abs"]
        assert float((lse - ref_lse).abs().max()) <= tol["lse"]

    # a call whose scratch would exceed the fixed array is refused, nothing enqueued
    big = pa.make_desc(65535, 64, 8, 128, 8192, 65536, 512, pa.PA_BF16, pa.PA_BF16, pa.PA_BF16)
    assert pa.workspace_size(big, 131072) > pa.NOALLOC_SCRATCH_BYTES
    nul = ctypes.c_void_p(0)
    st = pa._lib.paged_attn_decode_noalloc(nul, nul, nul, nul, nul, ctypes.c_float(0.1), nul,
                                           ctypes.byref(big), 131072, nul, nul, nul, nul, nul,
                                           nul)
    assert st == pa.PA_ERR_WORKSPACE
