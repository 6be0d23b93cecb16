"""int8 caches at the edges of the zero-point domain ([KVPaged] "KV quantization: FP8 and
INT8": one byte per element with a scale and a zero point; the library's reading: value =
(code - zero) * scale with codes and zero points in [-128, 127]).

Parity against the oracle with every code and zero points at both ends of the range (code -
zero reaches +-255), for decode on every kernel family (single pass and split) and for
prefill on both families. Zero points outside [-128, 127] are refused on the device: the
block is skipped, PA_DEVERR_ZERO is recorded, and the cache write leaves the row alone.
"""
import numpy as np
import pytest

import workloads
from oracle import attention
from tests.gpu_common import compare_decode

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

IMPLS = ["simt", "tc-grid", "tc-cta", "tc-warps"]


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_465_b200 as pa
    pa.set_decode_impl("auto")
    yield pa
    pa.set_decode_impl("auto")


class _Int8Pool:
    """A pool of random int8 codes (every code from -128 to 127 equally likely) whose blocks
    have zero points -128, 127 or a random in-range value, and sequences scattered over it."""

    def __init__(self, lens, B=16, Hq=32, Hkv=8, d=128, seed=7):
        rng = np.random.default_rng(seed)
        self.B, self.Hq, self.Hkv, self.d = B, Hq, Hkv, d
        self.lens = np.asarray(lens, np.int32)
        nblk = [-(-int(n) // B) for n in lens]
        self.NB = sum(nblk) + 8
        perm = rng.permutation(self.NB).astype(np.int32)
        self.mb = max(nblk)
        self.bt = np.full((len(lens), self.mb), -1, np.int32)
        o = 0
        for s, n in enumerate(nblk):
            self.bt[s, :n] = perm[o:o + n]
            o += n
        shape = (self.NB, Hkv, B, d)
        self.kc = rng.integers(-128, 128, shape).astype(np.int8)
        self.vc = rng.integers(-128, 128, shape).astype(np.int8)
        zchoice = np.array([-128, 127, -128, 127, 0], np.int32)
        self.kz = np.where(rng.random((self.NB, Hkv)) < 0.8,
                           zchoice[rng.integers(0, 5, (self.NB, Hkv))],
                           rng.integers(-128, 128, (self.NB, Hkv))).astype(np.int32)
        self.vz = np.where(rng.random((self.NB, Hkv)) < 0.8,
                           zchoice[rng.integers(0, 5, (self.NB, Hkv))],
                           rng.integers(-128, 128, (self.NB, Hkv))).astype(np.int32)
        # values (code - zero) * scale of a few units: scores of order one
        self.ks = (rng.uniform(0.5, 2.0, (self.NB, Hkv)) / 128).astype(np.float32)
        self.vs = (rng.uniform(0.5, 2.0, (self.NB, Hkv)) / 128).astype(np.float32)
        self.rng = rng
        self.scale = float(np.float32(1.0 / np.sqrt(d)))

    def dev(self):
        c = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()  # noqa: E731
        return dict(k_cache=c(self.kc), v_cache=c(self.vc), k_scales=c(self.ks),
                    v_scales=c(self.vs), k_zeros=c(self.kz), v_zeros=c(self.vz),
                    bt=c(self.bt), ctx=c(self.lens))

    def q(self, n):
        return workloads.bf16_bits_from_f32(
            self.rng.standard_normal((n, self.Hq, self.d), dtype=np.float32))


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


LENS = [1, 15, 16, 17, 300, 1000, 2049]


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("part", [0, 64, 512])
def test_decode_at_zero_point_extremes(pa, impl, part):
    p = _Int8Pool(LENS)
    g = p.dev()
    qb = p.q(len(LENS))
    ref_o, ref_l = attention.ref_decode(qb, p.kc, p.vc, p.bt, p.lens, p.scale, p.Hkv, "bf16",
                                        "int8", p.ks, p.vs, k_zeros=p.kz, v_zeros=p.vz)
    out = torch.empty((len(LENS), p.Hq, p.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((len(LENS), p.Hq), dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")
    pa.set_decode_impl(impl)
    try:
        pa.paged_attn_decode(_bf16_dev(qb), g["k_cache"], g["v_cache"], g["bt"], g["ctx"],
                             p.scale, out, max_context_len=int(p.lens.max()),
                             partition_size=part, k_scales=g["k_scales"],
                             v_scales=g["v_scales"], k_zeros=g["k_zeros"],
                             v_zeros=g["v_zeros"], lse_out=lse, workspace=ws)
        torch.cuda.synchronize()
        assert pa.device_error() == 0
    finally:
        pa.set_decode_impl("auto")
    compare_decode(out, lse, ref_o, ref_l, "int8")


@pytest.mark.parametrize("impl", ["auto", "simt"])
def test_prefill_at_zero_point_extremes(pa, impl):
    p = _Int8Pool(LENS, seed=8)
    g = p.dev()
    n = np.minimum(p.lens, [1, 15, 16, 9, 200, 130, 300]).astype(np.int32)
    qs = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    T = int(qs[-1])
    qb = p.q(T)
    ref_o, ref_l = attention.ref_prefill(qb, qs, p.kc, p.vc, p.bt, p.lens, p.scale, p.Hkv,
                                         "bf16", "int8", p.ks, p.vs, p.kz, p.vz)
    out = torch.empty((T, p.Hq, p.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, p.Hq), dtype=torch.float32, device="cuda")
    pa.set_decode_impl(impl)
    try:
        pa.paged_attn_prefill(_bf16_dev(qb), g["k_cache"], g["v_cache"], g["bt"], g["ctx"],
                              torch.from_numpy(qs).cuda(), p.scale, out,
                              max_query_len=int(n.max()), max_context_len=int(p.lens.max()),
                              k_scales=g["k_scales"], v_scales=g["v_scales"],
                              k_zeros=g["k_zeros"], v_zeros=g["v_zeros"], lse_out=lse)
        torch.cuda.synchronize()
        assert pa.device_error() == 0
    finally:
        pa.set_decode_impl("auto")
    compare_decode(out, lse, ref_o, ref_l, "int8")


@pytest.mark.parametrize("bad", [128, -129, 1 << 20])
def test_zero_point_out_of_range_is_flagged_everywhere(pa, bad):
    """One block of sequence 4 gets a K (then a V) zero point outside [-128, 127]: every
    decode family and both prefill families skip it and record PA_DEVERR_ZERO, with finite
    outputs; a cache write into that block leaves its rows alone and records the flag."""
    p = _Int8Pool(LENS, seed=9)
    blk = int(p.bt[4, 3])
    for which in ("k_zeros", "v_zeros"):
        g = p.dev()
        g[which][blk, 2] = bad
        qb = _bf16_dev(p.q(len(LENS)))
        out = torch.empty((len(LENS), p.Hq, p.d), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")
        assert pa.device_error() == 0
        for impl in IMPLS:
            for part in (0, 512):
                pa.set_decode_impl(impl)
                try:
                    pa.paged_attn_decode(qb, g["k_cache"], g["v_cache"], g["bt"], g["ctx"],
                                         p.scale, out, max_context_len=int(p.lens.max()),
                                         partition_size=part, k_scales=g["k_scales"],
                                         v_scales=g["v_scales"], k_zeros=g["k_zeros"],
                                         v_zeros=g["v_zeros"], workspace=ws)
                    assert pa.device_error() == pa.PA_DEVERR_ZERO, (impl, part)
                finally:
                    pa.set_decode_impl("auto")
                assert torch.isfinite(out.float()).all(), (impl, part)
        n = torch.tensor([1, 1, 1, 1, 64, 1, 1], dtype=torch.int32)
        qs = torch.cat([torch.zeros(1, dtype=torch.int32), torch.cumsum(n, 0).to(torch.int32)])
        T = int(qs[-1])
        qp = _bf16_dev(p.q(T))
        outp = torch.empty((T, p.Hq, p.d), dtype=torch.bfloat16, device="cuda")
        for impl in ("auto", "simt"):
            pa.set_decode_impl(impl)
            try:
                pa.paged_attn_prefill(qp, g["k_cache"], g["v_cache"], g["bt"], g["ctx"],
                                      qs.cuda(), p.scale, outp, max_query_len=64,
                                      max_context_len=int(p.lens.max()), k_scales=g["k_scales"],
                                      v_scales=g["v_scales"], k_zeros=g["k_zeros"],
                                      v_zeros=g["v_zeros"])
                assert pa.device_error() == pa.PA_DEVERR_ZERO, impl
            finally:
                pa.set_decode_impl("auto")
            assert torch.isfinite(outp.float()).all(), impl
        # the cache write: token 0 into the bad block, token 1 into a good one
        good = int(p.bt[5, 0])
        x = torch.randn(2, p.Hkv, p.d, device="cuda").to(torch.bfloat16)
        slots = torch.tensor([blk * p.B + 5, good * p.B + 5], dtype=torch.int64, device="cuda")
        kb, vb = g["k_cache"].clone(), g["v_cache"].clone()
        pa.reshape_and_cache(x, x, g["k_cache"], g["v_cache"], slots, k_scales=g["k_scales"],
                             v_scales=g["v_scales"], k_zeros=g["k_zeros"], v_zeros=g["v_zeros"])
        assert pa.device_error() == pa.PA_DEVERR_ZERO
        cache = g["k_cache"] if which == "k_zeros" else g["v_cache"]
        before = kb if which == "k_zeros" else vb
        assert torch.equal(cache[blk, 2], before[blk, 2])          # the bad (block, head)
        assert not torch.equal(cache[good, :, 5], before[good, :, 5])  # the good block written
