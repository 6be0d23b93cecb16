"""Seeded synthetic inputs for the paged decode-attention workloads.

This module is shared by the tests, the bench and the oracle's callers. It only DRAWS:
context lengths, the order of the physical block pool, query / key / value values, needle
positions, and the absmax statistic that the fp8 scale recipe is defined on. It holds none
of the method's arithmetic (no slot mapping, no block table, no cache write, no attention),
so neither the oracle nor the CUDA path takes any of its logic from the other through here.

Recipe (stated once, used everywhere):

* One ``numpy.random.Generator(PCG64(SeedSequence(seed)))`` per workload; the seed sequence
  is spawned into independent child streams in the fixed order
  ``[lens, pool, q, kv, needle]``; the ``kv`` stream is spawned again per sequence (and once
  more for a shared prefix), so any one sequence can be regenerated alone.
* Values are N(0, 1) drawn in float32. For bf16 inputs they are rounded to the nearest bf16
  (ties to even) and kept as uint16 bit patterns: the input *is* a bf16 tensor.
* ``pool_order`` is a permutation of the physical block ids; an allocator that hands blocks
  out in this order scatters every sequence across the pool.
* fp8 scales: per (sequence, logical block, kv head), ``absmax / 448`` over the bf16 values
  of the block's valid tokens (all ``d`` channels), separately for K and V, computed in
  float32; 1.0 where the absmax is 0. They are inputs of the fp8 cache write, not outputs.
* int8 scale / zero point: per (sequence, logical block, kv head), from the min and max of
  the same values: ``scale = (max - min) / 255`` and ``zero = rint(-128 - min / scale)``
  clipped to [-128, 127] (float32 arithmetic), so that min and max map to the ends of the
  int8 range; ``scale = 1, zero = 0`` where max == min.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import numpy as np

__all__ = ["Workload", "WORKLOADS", "Draw", "draw", "bf16_bits_from_f32"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and dtype recipe of one synthetic decode workload (one attention layer)."""

    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    kv_dtype: str  # "f32" | "bf16" | "fp8" | "int8"
    in_dtype: str  # dtype of q and of the new K/V handed to the cache write: "f32" | "bf16"
    lens: Tuple  # ("fixed", [..]) | ("uniform", lo, hi) | ("lognormal", median, sigma, lo, hi) | ("const", n)
    # split-KV partition in tokens; 0 = one pass per (seq, kv head); -1 = the library's choice
    partition_size: int = 0
    shared_prefix: Optional[Tuple[int, int]] = None  # (prefix tokens, suffix tokens per seq)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def out_dtype(self) -> str:
        return self.in_dtype

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # 4 seqs, ctx {5,16,17,40}, 4q/2kv, d 64, fp32, 32-block pool.
    "tiny": Workload("tiny", 0, 4, 4, 2, 64, 16, 32, "f32", "f32", ("fixed", [5, 16, 17, 40])),
    # 32 seqs, ctx ~ U{1..4096}, 32q/8kv, d 128, bf16, 8192-block pool; split chosen by the
    # library (too few (seq, kv head) pairs to keep every SM streaming in one pass).
    "b32": Workload("b32", 1, 32, 32, 8, 128, 16, 8192, "bf16", "bf16", ("uniform", 1, 4096),
                    partition_size=-1),
    # 100 seqs sharing a 200-token prefix + 50 private tokens, 32q/8kv, d 128, bf16.
    "shared": Workload("shared", 2, 100, 32, 8, 128, 16, 512, "bf16", "bf16", ("const", 250),
                       partition_size=-1, shared_prefix=(200, 50)),
    # 256 seqs, ctx lognormal(median 1024, sigma 1) clipped [16, 8192], fp8 KV, bf16 q/out.
    "b256": Workload("b256", 3, 256, 32, 8, 128, 16, 32768, "fp8", "bf16",
                     ("lognormal", 1024, 1.0, 16, 8192), partition_size=512),
    # the batch-256 workload with an int8 cache (scale + zero point per block and kv head)
    "b256_int8": Workload("b256_int8", 3, 256, 32, 8, 128, 16, 32768, "int8", "bf16",
                          ("lognormal", 1024, 1.0, 16, 8192), partition_size=512),
    # 8 seqs x 131072 tokens, 64q/8kv, d 128, bf16, split into 512-token partitions.
    "long": Workload("long", 4, 8, 64, 8, 128, 16, 65536, "bf16", "bf16", ("const", 131072),
                     partition_size=512),
}


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); return the uint16 bits.

    Used only to make the *inputs* bf16 tensors (the generator's data type), never by the
    method's own conversions.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    nan = np.isnan(x)
    # uint32 arithmetic cannot wrap for non-NaN inputs (they are below 0xFF800001)
    r = ((u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))) >> np.uint32(16)
         ).astype(np.uint16)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def _bits_to_f32(bits: np.ndarray) -> np.ndarray:
    bits = np.asarray(bits)
    return (bits.astype(np.uint32) << 16).view(np.float32)


class Draw:
    """All random inputs of one workload instance.

    ``context_lens[s]`` counts the token being decoded, whose K/V is the last row of
    ``kv(s)``. Arrays are float32 (``in_dtype == "f32"``) or uint16 bf16 bit patterns.
    """

    def __init__(self, wl: Workload, needle: bool = False, q_zero: bool = False,
                 lens_override: Optional[List[int]] = None,
                 q_scale: Optional[np.ndarray] = None):
        self.wl = wl
        self.needle = needle
        ss = np.random.SeedSequence(wl.seed)
        c_lens, c_pool, c_q, c_kv, c_needle = ss.spawn(5)
        self._kv_seq = c_kv.spawn(wl.num_seqs + 1)  # last child: shared prefix
        S, B = wl.num_seqs, wl.block_size
        rng = np.random.Generator(np.random.PCG64(c_lens))
        kind = wl.lens[0]
        if lens_override is not None:
            lens = np.asarray(lens_override, dtype=np.int64)
        elif kind == "fixed":
            lens = np.asarray(wl.lens[1], dtype=np.int64)
        elif kind == "const":
            lens = np.full(S, wl.lens[1], dtype=np.int64)
        elif kind == "uniform":
            lens = rng.integers(wl.lens[1], wl.lens[2] + 1, size=S)
        elif kind == "lognormal":
            med, sigma, lo, hi = wl.lens[1:]
            lens = np.clip(np.rint(np.exp(rng.normal(math.log(med), sigma, size=S))), lo, hi)
        else:
            raise ValueError(kind)
        self.context_lens = lens.astype(np.int32)
        assert self.context_lens.shape == (S,)
        prng = np.random.Generator(np.random.PCG64(c_pool))
        self.pool_order = prng.permutation(wl.num_blocks).astype(np.int32)
        qrng = np.random.Generator(np.random.PCG64(c_q))
        qf = qrng.standard_normal((S, wl.num_q_heads, wl.head_dim), dtype=np.float32)
        if q_zero:
            qf[:] = 0.0
        if q_scale is not None:     # per-(seq, head, channel) factors, broadcast over q
            qf = (qf * np.asarray(q_scale, dtype=np.float32)).astype(np.float32)
        self.q = self._typed(qf)
        # Needle: one token per (seq, kv head) whose key is c * (mean query of the group),
        # so that its logit dominates; its position is drawn uniformly over the context.
        nrng = np.random.Generator(np.random.PCG64(c_needle))
        self.needle_pos = np.stack(
            [nrng.integers(0, max(int(n), 1), size=wl.num_kv_heads) for n in self.context_lens])
        self._qf = self._as_f32(self.q)
        self._cache: Dict[int, Tuple[np.ndarray, np.ndarray]] = {}

    # -- typed storage of inputs ------------------------------------------------------
    def _typed(self, xf: np.ndarray) -> np.ndarray:
        return xf if self.wl.in_dtype == "f32" else bf16_bits_from_f32(xf)

    def _as_f32(self, x: np.ndarray) -> np.ndarray:
        return x if self.wl.in_dtype == "f32" else _bits_to_f32(x)

    def _draw_tokens(self, child: np.random.SeedSequence, n: int) -> Tuple[np.ndarray, np.ndarray]:
        wl = self.wl
        rng = np.random.Generator(np.random.PCG64(child))
        shape = (n, wl.num_kv_heads, wl.head_dim)
        k = rng.standard_normal(shape, dtype=np.float32)
        v = rng.standard_normal(shape, dtype=np.float32)
        return k, v

    def kv(self, s: int) -> Tuple[np.ndarray, np.ndarray]:
        """K and V of every token of sequence ``s`` (positions 0..ctx-1), [ctx, Hkv, d]."""
        if s in self._cache:
            return self._cache[s]
        wl = self.wl
        n = int(self.context_lens[s])
        if wl.shared_prefix is not None:
            p, sfx = wl.shared_prefix
            assert n == p + sfx
            kp, vp = self._draw_tokens(self._kv_seq[wl.num_seqs], p)
            ks, vs = self._draw_tokens(self._kv_seq[s], sfx)
            k, v = np.concatenate([kp, ks]), np.concatenate([vp, vs])
        else:
            k, v = self._draw_tokens(self._kv_seq[s], n)
        if self.needle and n > 0:
            G = wl.group
            qg = self._qf[s].reshape(wl.num_kv_heads, G, wl.head_dim).mean(axis=1)
            for h in range(wl.num_kv_heads):
                qn = qg[h] / max(float(np.linalg.norm(qg[h])), 1e-6)
                # logit of the needle ~ 12 / scale units above the N(0, d) background
                k[self.needle_pos[s, h], h] = qn * np.float32(12.0 * math.sqrt(wl.head_dim))
        out = (self._typed(k), self._typed(v))
        if len(self._cache) < 64:
            self._cache[s] = out
        return out

    def fp8_scales_logical(self, s: int) -> Tuple[np.ndarray, np.ndarray]:
        """Per (logical block, kv head) fp8 scales of sequence ``s``: absmax/448 (float32)."""
        wl = self.wl
        k, v = self.kv(s)
        n = int(self.context_lens[s])
        nb = -(-n // wl.block_size)
        out = []
        for x in (k, v):
            xf = np.abs(self._as_f32(x))
            pad = nb * wl.block_size - n
            if pad:
                xf = np.concatenate([xf, np.zeros((pad,) + xf.shape[1:], np.float32)])
            am = xf.reshape(nb, wl.block_size, wl.num_kv_heads, wl.head_dim).max(axis=(1, 3))
            sc = (am / np.float32(448.0)).astype(np.float32)
            sc[am == 0] = 1.0
            out.append(sc)
        return out[0], out[1]

    def int8_params_logical(self, s: int):
        """Per (logical block, kv head) int8 (k_scale, k_zero, v_scale, v_zero) of seq s."""
        wl = self.wl
        k, v = self.kv(s)
        n = int(self.context_lens[s])
        nb = -(-n // wl.block_size)
        res = []
        for x in (k, v):
            xf = self._as_f32(x)
            sc = np.ones((nb, wl.num_kv_heads), np.float32)
            zp = np.zeros((nb, wl.num_kv_heads), np.int32)
            for b in range(nb):
                blk = xf[b * wl.block_size:min(n, (b + 1) * wl.block_size)]
                for h in range(wl.num_kv_heads):
                    sc[b, h], zp[b, h] = _int8_params(blk[:, h, :])
            res += [sc, zp]
        return tuple(res)


def _int8_params(x: np.ndarray):
    """scale, zero of one block's values x (float32 array): min/max to the int8 range."""
    mn = np.float32(x.min())
    mx = np.float32(x.max())
    if mx <= mn:
        return np.float32(1.0), np.int32(0)
    scale = np.float32((mx - mn) / np.float32(255.0))
    zero = np.clip(np.rint(np.float32(-128.0) - mn / scale), -128, 127).astype(np.int32)
    return scale, zero


def draw(name_or_wl, **kw) -> Draw:
    wl = WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    return Draw(wl, **kw)


# ---------------------------------------------------------------------------------------
# prefill: a step that brings many new tokens per sequence
# ---------------------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    """Shape and length recipe of one synthetic prefill step (one attention layer).

    Sequence s holds context_lens[s] tokens after the step; the last query_lens[s] of them
    are the step's new tokens (their K/V are written, then they attend causally), the
    earlier ones were cached by earlier steps (a chunked prompt or a cached prefix).
    """

    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    kv_dtype: str
    in_dtype: str
    lens: Tuple       # context lengths, same forms as Workload.lens
    new: Tuple        # ("full",) every token new | ("chunk", n) the last min(n, ctx) tokens
                      # | ("uniform", lo, hi) a uniform count, at most ctx
    shared_prefix = None  # K/V of every sequence drawn independently

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def scaled(self, **kw) -> "PrefillWorkload":
        return dataclasses.replace(self, **kw)


PREFILL_WORKLOADS: Dict[str, PrefillWorkload] = {
    # 3 seqs: two whole prompts and a 7-token chunk after 33 cached tokens; fp32, d 64.
    "prefill_tiny": PrefillWorkload("prefill_tiny", 10, 3, 4, 2, 64, 16, 32, "f32", "f32",
                                    ("fixed", [5, 16, 40]), ("chunk", 16)),
    # 8 prompts of 2048 tokens prefilled whole: 32q/8kv, d 128, bf16.
    "prefill": PrefillWorkload("prefill", 11, 8, 32, 8, 128, 16, 8192, "bf16", "bf16",
                               ("const", 2048), ("full",)),
    # 16 sequences, 512-token chunks after cached contexts of U{512..3584}: 32q/8kv, bf16.
    "chunked": PrefillWorkload("chunked", 12, 16, 32, 8, 128, 16, 8192, "bf16", "bf16",
                               ("uniform", 1024, 4096), ("chunk", 512)),
    # the chunked recipe over an fp8-e4m3 cache (per-(block, kv head) scales)
    "chunked_fp8": PrefillWorkload("chunked_fp8", 12, 16, 32, 8, 128, 16, 8192, "fp8", "bf16",
                                   ("uniform", 1024, 4096), ("chunk", 512)),
}


class PrefillDraw(Draw):
    """All random inputs of one prefill step: lengths, pool order, q of the new tokens
    [T, Hq, d] (rows grouped by sequence), K/V of every context token of every sequence."""

    def __init__(self, wl: PrefillWorkload, lens_override: Optional[List[int]] = None,
                 new_override: Optional[List[int]] = None):
        self.wl = wl
        self.needle = False
        ss = np.random.SeedSequence(wl.seed)
        c_lens, c_pool, c_q, c_kv, c_new = ss.spawn(5)
        self._kv_seq = c_kv.spawn(wl.num_seqs + 1)
        S = wl.num_seqs
        rng = np.random.Generator(np.random.PCG64(c_lens))
        kind = wl.lens[0]
        if lens_override is not None:
            lens = np.asarray(lens_override, dtype=np.int64)
        elif kind == "fixed":
            lens = np.asarray(wl.lens[1], dtype=np.int64)
        elif kind == "const":
            lens = np.full(S, wl.lens[1], dtype=np.int64)
        elif kind == "uniform":
            lens = rng.integers(wl.lens[1], wl.lens[2] + 1, size=S)
        else:
            raise ValueError(kind)
        self.context_lens = lens.astype(np.int32)
        assert self.context_lens.shape == (S,)
        nrng = np.random.Generator(np.random.PCG64(c_new))
        if new_override is not None:
            qn = np.asarray(new_override, dtype=np.int64)
        elif wl.new[0] == "full":
            qn = lens.copy()
        elif wl.new[0] == "chunk":
            qn = np.minimum(lens, wl.new[1])
        elif wl.new[0] == "uniform":
            qn = np.minimum(lens, nrng.integers(wl.new[1], wl.new[2] + 1, size=S))
        else:
            raise ValueError(wl.new[0])
        assert np.all((qn >= 0) & (qn <= lens))
        self.query_lens = qn.astype(np.int32)
        self.query_start = np.concatenate([[0], np.cumsum(qn)]).astype(np.int32)
        prng = np.random.Generator(np.random.PCG64(c_pool))
        self.pool_order = prng.permutation(wl.num_blocks).astype(np.int32)
        qrng = np.random.Generator(np.random.PCG64(c_q))
        T = int(self.query_start[-1])
        self.q = self._typed(qrng.standard_normal((T, wl.num_q_heads, wl.head_dim),
                                                  dtype=np.float32))
        self._qf = None
        self._cache = {}

    @property
    def num_tokens(self) -> int:
        return int(self.query_start[-1])


def draw_prefill(name_or_wl, **kw) -> PrefillDraw:
    wl = PREFILL_WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    return PrefillDraw(wl, **kw)
