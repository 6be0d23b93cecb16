"""The allocation-free decode entry point, through the C ABI.

Some callers cannot allocate device memory: a plugin inside a host runtime that owns every
device allocation, a caller with no workspace argument to forward, a latency-bound loop
that must not risk cudaMalloc's implicit synchronisation. For them the library serves the
split-KV scratch from a fixed array of its own. The kernels are deterministic and the entry
point runs the same ones as the workspace entry point, so the check is bit identity of the
output and the lse, on calls in a row that find the previous call's leftovers in the shared
array: different shapes and dtypes, the tensor-core kernels (partitions merged in place by
the warp workers, and by the reduce kernel past 32 partitions) and the CUDA-core path. One
sequence per case comes from the oracle's draw and is checked against the oracle. A request
larger than the array is refused.
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


# (workload, context lengths or None, partition, kernel family, the sequence drawn from the
# oracle's inputs)
CASES = [
    (workloads.WORKLOADS["b256"].scaled(num_seqs=24), None, 512, "auto", 5),
    (workloads.WORKLOADS["long"].scaled(num_seqs=3), [9000, 700, 2500], 512, "auto", 1),
    (workloads.WORKLOADS["long"].scaled(num_seqs=3), [3000, 100, 2100], 64, "auto", 0),
    (workloads.WORKLOADS["b256"].scaled(num_seqs=24), None, 512, "simt", 7),
]


def test_noalloc_matches_workspace_entry_point_on_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_465_b200 as pa
    from paged_kv_cache_465_b200.scenario import DeviceScenario
    from oracle import flows
    from tests.gpu_common import compare_decode
    try:
        for wl, lens, part, impl, oseq in CASES:
            pa.set_decode_impl(impl)
            draw = workloads.draw(wl, lens_override=lens)
            sc = DeviceScenario(draw, draw_seqs=[oseq], partition_size=part)
            sc.step()  # cache write + decode through the workspace entry point
            torch.cuda.synchronize()
            assert pa.device_error() == 0
            ref_out, ref_lse = sc.out.clone(), sc.lse.clone()
            for _ in range(2):  # the second call finds the first one's scratch contents
                out = torch.full_like(sc.out, float("nan"))
                lse = torch.full_like(sc.lse, float("nan"))
                st, desc = _call_noalloc(pa, sc, out, lse)
                assert st == pa.PA_OK
                torch.cuda.synchronize()
                assert pa.device_error() == 0
                assert pa.workspace_size(desc, sc.max_context_len) > 0
                assert torch.equal(out, ref_out), (wl.name, impl, part)
                assert torch.equal(lse, ref_lse), (wl.name, impl, part)
            st_ref = flows.build_state(draw, write_seqs=[oseq])
            o_ref, l_ref = flows.ref_outputs(draw, st_ref, seqs=[oseq])
            compare_decode(out, lse, o_ref, l_ref, wl.kv_dtype, seqs=[oseq])
            del sc
    finally:
        pa.set_decode_impl("auto")

    # a call whose scratch would exceed the fixed array is refused, nothing enqueued
    big = pa.make_desc(65535, 64, 8, 128, 8192, 65536, 512, pa.PA_BF16, pa.PA_BF16, pa.PA_BF16)
    assert pa.workspace_size(big, 131072) > pa.NOALLOC_SCRATCH_BYTES
    nul = ctypes.c_void_p(0)
    st = pa._lib.paged_attn_decode_noalloc(nul, nul, nul, nul, nul, ctypes.c_float(0.1), nul,
                                           ctypes.byref(big), 131072, nul, nul, nul, nul, nul,
                                           nul)
    assert st == pa.PA_ERR_WORKSPACE
