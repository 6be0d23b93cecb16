"""GPU parity of the CUDA path against the oracle, through the C ABI (the Python binding).

Bit-exact: slot-mapped cache writes, block copies, cache contents after a whole workload.
Within the per-dtype tolerances of tests/gpu_common.py: decode outputs and lse, on the five
workloads (full size; the two largest on sampled sequences, in the launch configuration the
bench times), on both kernel families, on edge cases and needle variants. Bit-identical:
outputs under a different physical placement of the same logical KV, and shared-prefix
sequences against private unshared copies.
"""
import math

import numpy as np
import pytest

import workloads
from oracle import flows, paged as opaged, codecs
from tests.gpu_common import TOL, compare_decode, cache_codes, to_f64

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
    from paged_kv_cache_465_b200.scenario import DeviceScenario
    return DeviceScenario


def _bf16_dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).view(torch.int16).view(torch.bfloat16).cuda()


# ---------------------------------------------------------------------------------------
# cache write and block copy: bit-exact
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("in_dt,cache_dt,d", [("f32", "f32", 64), ("f32", "bf16", 128),
                                              ("bf16", "bf16", 128), ("bf16", "fp8", 128),
                                              ("f32", "fp8", 64), ("bf16", "bf16", 256),
                                              ("bf16", "int8", 128), ("f32", "int8", 64)])
def test_reshape_and_cache_bitexact(pa, in_dt, cache_dt, d):
    rng = np.random.default_rng(hash((in_dt, cache_dt, d)) % 2 ** 32)
    NB, H, B, T = 40, 4, 16, 300
    xf = (rng.standard_normal((T, H, d)) * rng.choice([1e-3, 1, 30, 700], (T, H, 1))).astype(np.float32)
    xin = xf if in_dt == "f32" else codecs.bf16_encode(xf)
    slots = rng.permutation(NB * B)[:T].astype(np.int64)
    slots[::17] = -1
    ks = rng.uniform(0.01, 2.0, (NB, H)).astype(np.float32)
    vs = rng.uniform(0.01, 2.0, (NB, H)).astype(np.float32)
    kz = rng.integers(-30, 31, (NB, H)).astype(np.int32)
    vz = rng.integers(-30, 31, (NB, H)).astype(np.int32)
    kref = opaged.new_cache(NB, H, B, d, cache_dt)
    vref = opaged.new_cache(NB, H, B, d, cache_dt)
    opaged.ref_reshape_and_cache(xin, xin[::-1].copy(), kref, vref, slots, in_dt, cache_dt, ks, vs,
                                 kz, vz)
    # device inputs: rows strided along T (a wider row buffer) to exercise k_stride
    tdt = torch.float32 if in_dt == "f32" else torch.bfloat16
    pad = 8
    wide = torch.zeros((T, H * d + pad), dtype=tdt)
    src = torch.from_numpy(xin) if in_dt == "f32" else torch.from_numpy(xin).view(torch.int16).view(torch.bfloat16)
    wide[:, :H * d] = src.reshape(T, H * d)
    k = wide.cuda()[:, :H * d].view(T, H, d)
    v = src.flip(0).contiguous().cuda()
    cdt = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.uint8,
           "int8": torch.int8}[cache_dt]
    kc = torch.zeros((NB, H, B, d), dtype=cdt, device="cuda")
    vc = torch.zeros_like(kc)
    sc = dict(k_scales=torch.from_numpy(ks).cuda(), v_scales=torch.from_numpy(vs).cuda()) \
        if cache_dt in ("fp8", "int8") else {}
    if cache_dt == "int8":
        sc.update(k_zeros=torch.from_numpy(kz).cuda(), v_zeros=torch.from_numpy(vz).cuda())
    pa.reshape_and_cache(k, v, kc, vc, torch.from_numpy(slots).cuda(), **sc)
    assert pa.device_error() == 0
    assert np.array_equal(cache_codes(kc), kref)
    assert np.array_equal(cache_codes(vc), vref)


def _fp8_write(pa, x, in_dt, scales, B=16, d=128):
    """Writes x [T, 1, d] (T a multiple of B) through reshape_and_cache into an fp8 cache,
    token t into slot t, and returns the GPU's codes and the oracle's."""
    T = x.shape[0]
    NB = T // B
    slots = np.arange(T, dtype=np.int64)
    kref = opaged.new_cache(NB, 1, B, d, "fp8")
    vref = opaged.new_cache(NB, 1, B, d, "fp8")
    opaged.ref_reshape_and_cache(x, x, kref, vref, slots, in_dt, "fp8", scales, scales)
    src = torch.from_numpy(x)
    if in_dt == "bf16":
        src = src.view(torch.int16).view(torch.bfloat16)
    k = src.cuda()
    kc = torch.zeros((NB, 1, B, d), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    sc = torch.from_numpy(scales).cuda()
    pa.reshape_and_cache(k, k, kc, vc, torch.from_numpy(slots).cuda(), k_scales=sc, v_scales=sc)
    assert pa.device_error() == 0
    return cache_codes(kc), kref


def _same_codes(got, ref):
    """Equal codes, except that a NaN may be either NaN pattern (S.1111.111)."""
    nan = (ref & 0x7F) == 0x7F
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.all((got[nan] & 0x7F) == 0x7F)


def test_fp8_write_every_bf16_value(pa):
    """All 65536 bf16 bit patterns (zeros, subnormals, normals, infinities, NaNs) through the
    fp8 cache write, with power-of-two and other block scales."""
    x = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(512, 1, 128)
    scales = np.array([[1.0], [0.5], [2.0 ** -8], [3.0], [0.37], [2.0 ** 6], [1e-3], [7.25]] * 4,
                      np.float32)
    got, ref = _fp8_write(pa, x, "bf16", scales)
    _same_codes(got, ref)


def test_fp8_write_rounding_midpoints(pa):
    """float32 inputs at every midpoint between adjacent E4M3 magnitudes (ties to even), one
    float32 step either side of it, past the largest finite value (saturation), and the
    specials; block scales 1 and 2^-3 (x / scale exact), 0.3 (rounded division)."""
    mags = codecs.E4M3_TABLE[:127]
    mids = ((mags[1:] + mags[:-1]) / 2).astype(np.float32)
    vals = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
                           mags.astype(np.float32),
                           np.array([448, 460, 464, 464.0001, 480, 1e30, np.inf, np.nan, 0.0,
                                     1e-45, 2.0 ** -10, 3 * 2.0 ** -10], np.float32)])
    vals = np.concatenate([vals, -vals]).astype(np.float32)
    per = 16 * 128
    n_blocks = -(-vals.size // per)
    x = np.zeros(n_blocks * per, np.float32)
    x[:vals.size] = vals
    for sc in (1.0, 0.125, 0.3):
        scales = np.full((n_blocks, 1), sc, np.float32)
        got, ref = _fp8_write(pa, (x * np.float32(sc)).astype(np.float32).reshape(-1, 1, 128),
                              "f32", scales)
        _same_codes(got, ref)


def test_int8_write_ties_and_clipping(pa):
    """int8 cache write at every half-integer x / scale in [-200, 200] (ties to even before
    the zero point is added), one float32 step either side, and values past the byte's
    range, with several zero points and scales (1 and 0.5 keep x / scale exact)."""
    B, d = 16, 128
    base = np.arange(-200, 200, dtype=np.float64) + 0.5
    vals = np.concatenate([base, np.nextafter(base.astype(np.float32), np.float32(-1e9)),
                           np.nextafter(base.astype(np.float32), np.float32(1e9)),
                           np.array([0.0, -0.0, 1e9, -1e9, 127.5, -128.5, 127.49998], np.float32)])
    vals = vals.astype(np.float32)
    per = B * d
    NB = -(-vals.size // per) * 4
    x = np.zeros((NB * per,), np.float32)
    reps = NB // (-(-vals.size // per))
    for r in range(reps):
        x[r * (NB // reps) * per: r * (NB // reps) * per + vals.size] = vals
    zeros = np.array([[0], [7], [-30], [100]] * (NB // 4), np.int32)[:NB]
    for sc in (1.0, 0.5):
        scales = np.full((NB, 1), sc, np.float32)
        xs = (x * np.float32(sc)).astype(np.float32).reshape(-1, 1, d)
        T = xs.shape[0]
        slots = np.arange(T, dtype=np.int64)
        kref = opaged.new_cache(NB, 1, B, d, "int8")
        vref = opaged.new_cache(NB, 1, B, d, "int8")
        opaged.ref_reshape_and_cache(xs, xs, kref, vref, slots, "f32", "int8", scales, scales,
                                     zeros, zeros)
        k = torch.from_numpy(xs).cuda()
        kc = torch.zeros((NB, 1, B, d), dtype=torch.int8, device="cuda")
        vc = torch.zeros_like(kc)
        s_d = torch.from_numpy(scales).cuda()
        z_d = torch.from_numpy(zeros).cuda()
        pa.reshape_and_cache(k, k, kc, vc, torch.from_numpy(slots).cuda(), k_scales=s_d,
                             v_scales=s_d, k_zeros=z_d, v_zeros=z_d)
        assert pa.device_error() == 0
        assert np.array_equal(cache_codes(kc), kref)


@pytest.mark.parametrize("cache_dt", ["f32", "bf16", "fp8", "int8"])
def test_copy_blocks_bitexact(pa, cache_dt):
    rng = np.random.default_rng(5)
    NB, H, B, d = 64, 8, 16, 128
    store = {"f32": np.float32, "bf16": np.uint16, "fp8": np.uint8, "int8": np.int8}[cache_dt]
    if cache_dt == "f32":
        k0 = rng.standard_normal((NB, H, B, d)).astype(np.float32)
        v0 = rng.standard_normal((NB, H, B, d)).astype(np.float32)
    else:
        lo, hi = {"bf16": (0, 2 ** 16), "fp8": (0, 256), "int8": (-128, 128)}[cache_dt]
        k0 = rng.integers(lo, hi, (NB, H, B, d)).astype(store)
        v0 = rng.integers(lo, hi, (NB, H, B, d)).astype(store)
    quant = cache_dt in ("fp8", "int8")
    ks0 = rng.uniform(size=(NB, H)).astype(np.float32)
    vs0 = rng.uniform(size=(NB, H)).astype(np.float32)
    kz0 = rng.integers(-128, 128, (NB, H)).astype(np.int32)
    vz0 = rng.integers(-128, 128, (NB, H)).astype(np.int32)
    srcs = rng.choice(NB, 20, replace=False)
    dsts = rng.choice(np.setdiff1d(np.arange(NB), srcs), 20, replace=False)
    pairs = [(int(s), int(t)) for s, t in zip(srcs, dsts)]
    kr, vr, ksr, vsr, kzr, vzr = k0.copy(), v0.copy(), ks0.copy(), vs0.copy(), kz0.copy(), vz0.copy()
    opaged.ref_copy_blocks(kr, vr, pairs, ksr if quant else None, vsr if quant else None,
                           kzr if cache_dt == "int8" else None, vzr if cache_dt == "int8" else None)

    def dev(x):
        t = torch.from_numpy(x)
        if cache_dt == "bf16":
            t = t.view(torch.int16).view(torch.bfloat16)
        return t.cuda()
    kc, vc = dev(k0), dev(v0)
    ksd, vsd = torch.from_numpy(ks0).cuda(), torch.from_numpy(vs0).cuda()
    kzd, vzd = torch.from_numpy(kz0).cuda(), torch.from_numpy(vz0).cuda()
    pa.copy_blocks(kc, vc, torch.tensor(pairs, dtype=torch.int32, device="cuda"),
                   k_scales=ksd if quant else None, v_scales=vsd if quant else None,
                   k_zeros=kzd if cache_dt == "int8" else None,
                   v_zeros=vzd if cache_dt == "int8" else None)
    assert pa.device_error() == 0
    assert np.array_equal(cache_codes(kc), kr) and np.array_equal(cache_codes(vc), vr)
    assert np.array_equal(ksd.cpu().numpy(), ksr) and np.array_equal(vsd.cpu().numpy(), vsr)
    assert np.array_equal(kzd.cpu().numpy(), kzr) and np.array_equal(vzd.cpu().numpy(), vzr)


# ---------------------------------------------------------------------------------------
# whole workloads
# ---------------------------------------------------------------------------------------
def _run_and_compare(pa, scen, draw, impl="auto", draw_seqs=None, partition_size=None,
                     check_cache=True, shared=True):
    pa.set_decode_impl(impl)
    try:
        sc = scen(draw, draw_seqs=draw_seqs, partition_size=partition_size, shared=shared)
        sc.step()
        torch.cuda.synchronize()
        assert pa.device_error() == 0
        st = flows.build_state(draw, write_seqs=draw_seqs, shared=shared)
        seqs = sorted(sc.draw_seqs)
        out_ref, lse_ref = flows.ref_outputs(draw, st, seqs=seqs)
        stats = compare_decode(sc.out, sc.lse, out_ref, lse_ref, draw.wl.kv_dtype, seqs=seqs)
        if check_cache:
            assert np.array_equal(sc.block_tables.cpu().numpy(), st.block_tables)
            assert np.array_equal(cache_codes(sc.cache.k_cache), st.k_cache)
            assert np.array_equal(cache_codes(sc.cache.v_cache), st.v_cache)
        return sc, stats
    finally:
        pa.set_decode_impl("auto")


@pytest.mark.parametrize("impl", ["simt", "auto"])
def test_tiny_workload(pa, scen, impl):
    d = workloads.draw("tiny")
    _run_and_compare(pa, scen, d, impl)
    # the four decode tokens land at offsets 4, 15, 0 (a new block) and 7
    sc = scen(d)
    offs = (sc.step_slots.cpu().numpy() % 16).tolist()
    assert offs == [4, 15, 0, 7]


SPLIT_IMPLS = ["simt", "tc-grid", "tc-cta", "tc-warps"]


@pytest.mark.parametrize("impl", SPLIT_IMPLS)
@pytest.mark.parametrize("part", [0, 512, -1])   # -1: the library chooses the split
def test_batch32_workload(pa, scen, impl, part):
    _run_and_compare(pa, scen, workloads.draw("b32"), impl, partition_size=part)


@pytest.mark.parametrize("impl", ["simt", "auto"])
def test_shared_prefix_workload(pa, scen, impl):
    d = workloads.draw("shared")
    sc, _ = _run_and_compare(pa, scen, d, impl)
    assert len(sc.cow_pairs) == 99
    assert sc.cache.num_blocks - sc.cache.alloc.num_free() == 412
    # shared-prefix sequences == private unshared copies, bit for bit
    pa.set_decode_impl(impl)
    try:
        un = scen(d, shared=False)
        un.step()
        torch.cuda.synchronize()
        assert torch.equal(un.out, sc.out) and torch.equal(un.lse, sc.lse)
    finally:
        pa.set_decode_impl("auto")


@pytest.mark.parametrize("impl", SPLIT_IMPLS)
@pytest.mark.parametrize("part", [512, 0])
@pytest.mark.parametrize("name", ["b256", "b256_int8"])
def test_batch256_full_size_sampled(pa, scen, impl, part, name):
    d = workloads.draw(name)
    lens = d.context_lens
    sample = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 7, 100, 200, 255})
    _run_and_compare(pa, scen, d, impl, draw_seqs=sample, partition_size=part, check_cache=False)


@pytest.mark.parametrize("impl", ["auto", "tc-cta"])
def test_long_context_full_size_sampled(pa, scen, impl):
    d = workloads.draw("long")
    _run_and_compare(pa, scen, d, impl, draw_seqs=[5], check_cache=False)


# ---------------------------------------------------------------------------------------
# invariances, needles, closed forms, edge cases
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("impl", SPLIT_IMPLS)
@pytest.mark.parametrize("name,part", [("b32", 0), ("b32", 512), ("b32", -1), ("b256", 512),
                                       ("b256_int8", 512), ("shared", -1)])
def test_physical_placement_bit_identical(pa, scen, impl, name, part):
    wl = workloads.WORKLOADS[name].scaled(num_seqs=6)
    pa.set_decode_impl(impl)
    try:
        d1 = workloads.draw(wl)
        s1 = scen(d1, partition_size=part)
        s1.step()
        d2 = workloads.draw(wl)
        d2.pool_order = np.roll(d2.pool_order[::-1], 7).copy()
        s2 = scen(d2, partition_size=part)
        s2.step()
        torch.cuda.synchronize()
        assert not torch.equal(s1.block_tables, s2.block_tables)
        assert torch.equal(s1.out, s2.out) and torch.equal(s1.lse, s2.lse)
    finally:
        pa.set_decode_impl("auto")


@pytest.mark.parametrize("impl", SPLIT_IMPLS)
@pytest.mark.parametrize("name,part,lens", [
    ("b32", 0, [1, 2, 15, 16, 17, 31, 33, 4096]),
    ("b32", 512, [511, 512, 513, 1024, 1025, 3000]),
    ("b32", -1, [1, 2, 15, 16, 17, 31, 33, 64, 65, 4096]),
    ("b256", 512, [16, 17, 500, 512, 2049, 8192]),
    ("b256", 0, [1, 16, 100, 8192]),
    ("b256_int8", 512, [16, 17, 500, 513, 2049]),
    ("long", 512, [20000, 513]),
])
def test_ragged_lengths_and_needles(pa, scen, impl, name, part, lens):
    wl = workloads.WORKLOADS[name].scaled(num_seqs=len(lens))
    for needle in (False, True):
        d = workloads.draw(wl, lens_override=lens, needle=needle)
        _run_and_compare(pa, scen, d, impl, partition_size=part)


@pytest.mark.parametrize("impl", SPLIT_IMPLS)
@pytest.mark.parametrize("part", [512, 0])
def test_fp8_query_dynamic_range(pa, scen, impl, part):
    """fp8 cache, q with a wide range of magnitudes: the heads of a group 2^-8, 2^-4, 1 and
    2 apart and every channel scaled by 2^u, u uniform in [-12, 3] (bf16 inputs), with and
    without a needle. The tensor-core kernels take the K codes into 8-bit products against
    q split into two E4M3 codes per element under a power of two per head; this is the
    case where one power of two per group, or one E4M3 code per element, would fail."""
    lens = [16, 17, 500, 700, 1500, 2049]
    wl = workloads.WORKLOADS["b256"].scaled(num_seqs=len(lens))
    assert wl.kv_dtype == "fp8" and wl.group == 4
    rng = np.random.default_rng(465)
    head = 2.0 ** np.array([-8, -4, 0, 1] * (wl.num_q_heads // 4))
    chan = 2.0 ** rng.uniform(-12.0, 3.0, size=(len(lens), wl.num_q_heads, wl.head_dim))
    scale = (head[None, :, None] * chan).astype(np.float32)
    for needle in (False, True):
        d = workloads.draw(wl, lens_override=lens, needle=needle, q_scale=scale)
        _run_and_compare(pa, scen, d, impl, partition_size=part)


@pytest.mark.parametrize("impl", ["simt", "auto"])
def test_zero_query_is_mean_of_values(pa, scen, impl):
    wl = workloads.WORKLOADS["b32"].scaled(num_seqs=3)
    d = workloads.draw(wl, q_zero=True, lens_override=[5, 300, 1000])
    sc, _ = _run_and_compare(pa, scen, d, impl)
    out = to_f64(sc.out)
    for s in range(3):
        k, v = d.kv(s)
        vm = codecs.bf16_decode(v).mean(axis=0)      # [Hkv, d]
        G = wl.group
        for h in range(wl.num_q_heads):
            assert np.abs(out[s, h] - vm[h // G]).max() < TOL["bf16"]["max_abs"]
        assert np.allclose(to_f64(sc.lse)[s], math.log(d.context_lens[s]), atol=1e-3)


@pytest.mark.parametrize("impl", SPLIT_IMPLS)
@pytest.mark.parametrize("hq,hkv,dim,kv", [(8, 8, 128, "bf16"), (16, 8, 128, "bf16"),
                                            (64, 4, 128, "bf16"), (16, 2, 64, "bf16"),
                                            (8, 1, 256, "bf16"), (32, 8, 128, "fp8"),
                                            (64, 8, 128, "fp8"), (8, 2, 128, "f32"),
                                            (6, 2, 128, "bf16"), (32, 8, 128, "int8"),
                                            (8, 8, 128, "int8"), (16, 2, 64, "int8")])
def test_head_shapes(pa, scen, impl, hq, hkv, dim, kv):
    in_dt = "f32" if kv == "f32" else "bf16"
    wl = workloads.Workload("shape", 9, 5, hq, hkv, dim, 16, 512, kv, in_dt,
                            ("fixed", [1, 17, 100, 700, 1500]))
    for part in (0, 256, 1024):
        _run_and_compare(pa, scen, workloads.draw(wl), impl, partition_size=part)


def test_empty_context_and_error_flags(pa):
    S, Hq, Hkv, d, NB = 3, 8, 2, 128, 16
    q = torch.randn(S, Hq, d, device="cuda").to(torch.bfloat16)
    kc = torch.randn(NB, Hkv, 16, d, device="cuda").to(torch.bfloat16)
    vc = torch.randn(NB, Hkv, 16, d, device="cuda").to(torch.bfloat16)
    bt = torch.tensor([[0, 1], [2, -1], [3, 4]], dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty(S, Hq, device="cuda")
    assert pa.device_error() == 0
    for part in (0, 16):
        ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
        pa.paged_attn_decode(q, kc, vc, bt, torch.tensor([0, 5, 0], dtype=torch.int32,
                                                         device="cuda"),
                             0.1, out, max_context_len=32, partition_size=part, lse_out=lse,
                             workspace=ws)
        torch.cuda.synchronize()
        assert pa.device_error() == 0
        assert torch.all(out[0] == 0) and torch.all(out[2] == 0)
        assert torch.all(torch.isneginf(lse[0])) and torch.all(torch.isfinite(lse[1]))
    # an out-of-range block id is skipped and flagged, never dereferenced
    bad = torch.tensor([[0, 1_000_000], [2, -1], [3, 4]], dtype=torch.int32, device="cuda")
    for part in (0, 16):
        ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
        pa.paged_attn_decode(q, kc, vc, bad, torch.tensor([20, 5, 30], dtype=torch.int32,
                                                          device="cuda"),
                             0.1, out, max_context_len=32, partition_size=part, workspace=ws)
        assert pa.device_error() & pa.PA_DEVERR_BLOCK_ID
        assert pa.device_error() == 0
        assert torch.isfinite(out[2].float()).all()
    # a context longer than max_context_len is clamped and flagged
    pa.paged_attn_decode(q, kc, vc, bt, torch.tensor([20, 5, 40], dtype=torch.int32,
                                                     device="cuda"),
                         0.1, out, max_context_len=32)
    assert pa.device_error() & pa.PA_DEVERR_CONTEXT
    # a slot past the pool and a copy pair past the pool are skipped and flagged
    k1 = torch.randn(2, Hkv, d, device="cuda").to(torch.bfloat16)
    before = kc.clone()
    pa.reshape_and_cache(k1, k1, kc, vc, torch.tensor([5, NB * 16 + 3], dtype=torch.int64,
                                                      device="cuda"))
    assert pa.device_error() & pa.PA_DEVERR_SLOT
    assert torch.equal(kc[1:], before[1:]) and torch.equal(kc[0, :, 6:], before[0, :, 6:])
    pa.copy_blocks(kc, vc, torch.tensor([[0, NB]], dtype=torch.int32, device="cuda"))
    assert pa.device_error() & pa.PA_DEVERR_PAIR


# ---------------------------------------------------------------------------------------
# block sizes 8 and 32 ("the block-size knob"; Theorem 1 trade-off note)
# ---------------------------------------------------------------------------------------
def _bs(name, B, **kw):
    wl = workloads.WORKLOADS[name]
    return wl.scaled(block_size=B, num_blocks=wl.num_blocks * 16 // B, **kw)


@pytest.mark.parametrize("B", [8, 32])
@pytest.mark.parametrize("impl", ["simt", "auto"])
def test_block_sizes_tiny_and_shared(pa, scen, B, impl):
    _run_and_compare(pa, scen, workloads.draw(_bs("tiny", B)), impl)
    d = workloads.draw(_bs("shared", B, num_seqs=20))
    sc, _ = _run_and_compare(pa, scen, d, impl)
    # a 200-token prefix fills 25 blocks of 8 exactly (nothing to copy); with 32-token
    # blocks its last block holds 8 tokens and every child copies it before appending
    assert len(sc.cow_pairs) == (0 if B == 8 else 19)


@pytest.mark.parametrize("impl", SPLIT_IMPLS)
@pytest.mark.parametrize("B", [8, 32])
@pytest.mark.parametrize("name,part,seqs", [("b32", 0, 32), ("b32", 512, 32), ("b32", -1, 32),
                                            ("b256", 512, 12), ("b256", 0, 6),
                                            ("b256_int8", 512, 12)])
def test_block_sizes_workloads(pa, scen, impl, B, name, part, seqs):
    _run_and_compare(pa, scen, workloads.draw(_bs(name, B, num_seqs=seqs)), impl,
                     partition_size=part)


@pytest.mark.parametrize("impl", SPLIT_IMPLS)
@pytest.mark.parametrize("B", [8, 32])
@pytest.mark.parametrize("name,part", [("b32", 0), ("b32", 512), ("b256", 512),
                                       ("b256_int8", 512)])
def test_block_sizes_ragged_needles_and_placement(pa, scen, impl, B, name, part):
    lens = [1, 7, 8, 9, 15, 16, 17, 24, 31, 32, 33, 40, 511, 513, 1000]
    wl = _bs(name, B, num_seqs=len(lens))
    for needle in (False, True):
        _run_and_compare(pa, scen, workloads.draw(wl, lens_override=lens, needle=needle), impl,
                         partition_size=part)
    pa.set_decode_impl(impl)
    try:
        d1 = workloads.draw(wl, lens_override=lens)
        s1 = scen(d1, partition_size=part)
        s1.step()
        d2 = workloads.draw(wl, lens_override=lens)
        d2.pool_order = np.roll(d2.pool_order[::-1], 5).copy()
        s2 = scen(d2, partition_size=part)
        s2.step()
        torch.cuda.synchronize()
        assert not torch.equal(s1.block_tables, s2.block_tables)
        assert torch.equal(s1.out, s2.out) and torch.equal(s1.lse, s2.lse)
    finally:
        pa.set_decode_impl("auto")


@pytest.mark.parametrize("impl", SPLIT_IMPLS)
@pytest.mark.parametrize("B", [8, 32])
@pytest.mark.parametrize("hq,hkv,dim,kv", [(64, 4, 128, "bf16"), (8, 1, 256, "bf16"),
                                            (32, 8, 128, "fp8"), (16, 2, 64, "int8"),
                                            (8, 2, 128, "f32")])
def test_block_sizes_head_shapes(pa, scen, impl, B, hq, hkv, dim, kv):
    in_dt = "f32" if kv == "f32" else "bf16"
    wl = workloads.Workload("shape", 9, 5, hq, hkv, dim, B, 8192 // B, kv, in_dt,
                            ("fixed", [1, 9, 100, 700, 1500]))
    for part in (0, 256, 1024):
        _run_and_compare(pa, scen, workloads.draw(wl), impl, partition_size=part)


@pytest.mark.parametrize("impl", SPLIT_IMPLS)
def test_block_size_8_bad_second_half_is_flagged(pa, impl):
    """A 16-token sub-tile of 8-token blocks whose second block id is out of range: that
    block is skipped and flagged, the rest of the context still decodes."""
    S, Hq, Hkv, d, B, NB = 2, 8, 2, 128, 8, 16
    q = torch.randn(S, Hq, d, device="cuda").to(torch.bfloat16)
    kc = torch.randn(NB, Hkv, B, d, device="cuda").to(torch.bfloat16)
    vc = torch.randn(NB, Hkv, B, d, device="cuda").to(torch.bfloat16)
    bt = torch.tensor([[0, 1_000_000, 2, 3], [4, 5, 6, 7]], dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    pa.set_decode_impl(impl)
    try:
        for part in (0, 16):
            ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
            pa.paged_attn_decode(q, kc, vc, bt, torch.tensor([30, 30], dtype=torch.int32,
                                                             device="cuda"),
                                 0.1, out, max_context_len=32, partition_size=part,
                                 workspace=ws)
            assert pa.device_error() & pa.PA_DEVERR_BLOCK_ID
            assert pa.device_error() == 0
            assert torch.isfinite(out.float()).all()
    finally:
        pa.set_decode_impl("auto")
