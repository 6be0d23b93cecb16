"""Python binding of libpagedattn.so (paged decode attention for B200, sm_100a).

Thin ctypes marshalling over the C ABI declared in ``include/pagedattn.h``: every function
here checks tensor devices, dtypes, shapes and contiguity, turns tensors into device
pointers and forwards to the library with torch's current CUDA stream. All device work runs
in the library's own kernels; there is no fallback of any kind. Importing this package
raises if the compiled library is missing (build it with
``python paged_kv_cache_465_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python paged_kv_cache_465_b200/build.py` "
        "(nvcc, sm_100a). There is no non-CUDA implementation.")

_lib = ctypes.CDLL(LIB_PATH)

# ---------------------------------------------------------------------------------------
# enums (mirror include/pagedattn.h)
# ---------------------------------------------------------------------------------------
PA_F32, PA_BF16, PA_FP8_E4M3, PA_INT8 = 0, 1, 2, 3
PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_NO_BLOCKS, PA_ERR_WORKSPACE, \
    PA_ERR_DEVICE = 0, -1, -2, -3, -4, -5, -6
PA_DEVERR_BLOCK_ID, PA_DEVERR_SLOT, PA_DEVERR_PAIR, PA_DEVERR_CONTEXT, PA_DEVERR_TIMEOUT = \
    0x1, 0x2, 0x4, 0x8, 0x10
PA_DEVERR_QUERY = 0x20
PA_DEVERR_ZERO = 0x40
_STATUS = {0: "PA_OK", -1: "PA_ERR_INVALID", -2: "PA_ERR_UNSUPPORTED", -3: "PA_ERR_CUDA",
           -4: "PA_ERR_NO_BLOCKS", -5: "PA_ERR_WORKSPACE", -6: "PA_ERR_DEVICE"}


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_STATUS.get(status, status)}")
        self.status = status


class NoBlocks(PagedAttnError):
    """The allocator's free queue is short; the call changed nothing."""


class pa_decode_desc(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int), ("num_q_heads", ctypes.c_int),
                ("num_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("block_size", ctypes.c_int), ("max_blocks_per_seq", ctypes.c_int),
                ("num_blocks", ctypes.c_int), ("partition_size", ctypes.c_int),
                ("q_dtype", ctypes.c_int), ("kv_dtype", ctypes.c_int),
                ("out_dtype", ctypes.c_int)]


_vp, _i, _i64, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_P = ctypes.POINTER
_SIGS = {
    "pa_version": (ctypes.c_char_p, []),
    "paged_attn_workspace_size": (_sz, [_P(pa_decode_desc), _i]),
    "paged_attn_decode_launches": (_i, [_P(pa_decode_desc), _i]),
    "paged_attn_partition_size": (_i, [_P(pa_decode_desc), _i]),
    "paged_attn_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _P(pa_decode_desc), _i, _vp,
                               _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "paged_attn_decode_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp, _P(pa_decode_desc), _i,
                                       _vp, _vp, _vp, _vp, _vp, _vp]),
    "paged_attn_prefill": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _f, _vp,
                                _P(pa_decode_desc), _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "reshape_and_cache": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i64, _i64, _i, _i, _i, _i, _i, _i,
                               _vp, _vp, _vp, _vp, _vp]),
    "copy_blocks": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "pa_device_error": (_i, [_P(_i), _vp]),
    "pa_alloc_create": (_vp, [_i, _i]),
    "pa_alloc_create_ordered": (_vp, [_i, _i, _vp]),
    "pa_alloc_destroy": (None, [_vp]),
    "pa_alloc_num_free": (_i, [_vp]),
    "pa_alloc_ref_count": (_i, [_vp, _i]),
    "pa_alloc_add_seq": (_i, [_vp, _i, _i, _vp]),
    "pa_alloc_fork": (_i, [_vp, _i, _i]),
    "pa_alloc_append": (_i, [_vp, _i, _i, _vp, _vp, _P(_i)]),
    "pa_alloc_append_batch": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _P(_i)]),
    "pa_alloc_free_seq": (_i, [_vp, _i]),
    "pa_alloc_block_table": (_i, [_vp, _i, _vp, _i]),
    "pa_alloc_seq_len": (_i, [_vp, _i]),
    "pa_alloc_free_queue": (_i, [_vp, _vp, _i]),
    "pa_set_decode_impl": (_i, [_i]),
    "pa_alloc_add_seq_tokens": (_i, [_vp, _i, _vp, _i, _vp, _P(_i)]),
    "pa_alloc_num_cached": (_i, [_vp]),
    "pa_alloc_cache_stats": (_i, [_vp, _P(_i64), _P(_i64)]),
    "pa_alloc_block_hash": (_i, [_vp, _i, _vp]),
    "pa_sha256": (None, [_vp, _sz, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def version() -> str:
    return _lib.pa_version().decode()


def _check(st: int, what: str) -> None:
    if st == PA_ERR_NO_BLOCKS:
        raise NoBlocks(st, what)
    if st != PA_OK:
        raise PagedAttnError(st, what)


# ---------------------------------------------------------------------------------------
# torch plumbing (device memory and streams only)
# ---------------------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t == torch.float32:
        return PA_F32
    if t == torch.bfloat16:
        return PA_BF16
    if t in (torch.float8_e4m3fn, torch.uint8):
        return PA_FP8_E4M3
    if t == torch.int8:
        return PA_INT8
    raise TypeError(f"unsupported dtype {t}")


def _dev(x, name, dtype=None, contiguous=True):
    if x is None:
        return None
    if not getattr(x, "is_cuda", False):
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and x.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {x.dtype}, expected {dtype}")
    if contiguous and not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(x.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


DECODE_IMPLS = {"auto": 0, "simt": 1, "tc": 2, "tc-grid": 3, "tc-cta": 4, "tc-warps": 5}


def set_decode_impl(impl: str = "auto") -> None:
    """Chooses the decode kernels: "auto" (tensor cores where supported), "simt" (CUDA-core
    fp32 path everywhere), "tc" (tensor cores, automatic kernel), or a fixed tensor-core
    kernel: "tc-grid" (one CTA per work item), "tc-cta" (persistent CTAs), "tc-warps"
    (persistent warp workers) where the call allows it."""
    code = DECODE_IMPLS[impl]
    _check(_lib.pa_set_decode_impl(code), "pa_set_decode_impl")


def make_desc(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, num_blocks,
              partition_size, q_dtype, kv_dtype, out_dtype, block_size=16) -> pa_decode_desc:
    return pa_decode_desc(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                          max_blocks_per_seq, num_blocks, partition_size, q_dtype, kv_dtype,
                          out_dtype)


def workspace_size(desc: pa_decode_desc, max_context_len: int) -> int:
    return int(_lib.paged_attn_workspace_size(ctypes.byref(desc), int(max_context_len)))


PARTITION_AUTO = -1  # partition_size: the library chooses the split (PA_PARTITION_AUTO)


def partition_size_for(desc: pa_decode_desc, max_context_len: int) -> int:
    """The partition (tokens, 0 = one pass) a decode call with this descriptor uses."""
    return int(_lib.paged_attn_partition_size(ctypes.byref(desc), int(max_context_len)))


def decode_launches(desc: pa_decode_desc, max_context_len: int) -> int:
    """Kernel launches of one paged_attn_decode call with this descriptor (current impl)."""
    return int(_lib.paged_attn_decode_launches(ctypes.byref(desc), int(max_context_len)))


def decode_desc_for(q, k_cache, block_tables, partition_size: int) -> pa_decode_desc:
    S, Hq, d = q.shape
    NB, Hkv, B, d2 = k_cache.shape
    if d2 != d:
        raise ValueError("head_dim of q and cache differ")
    qd = _dtype_code(q.dtype)
    return make_desc(S, Hq, Hkv, d, block_tables.shape[1], NB, partition_size, qd,
                     _dtype_code(k_cache.dtype), qd, block_size=B)


def paged_attn_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, out, *,
                      max_context_len: int, partition_size: int = 0, k_scales=None,
                      v_scales=None, k_zeros=None, v_zeros=None, lse_out=None, workspace=None,
                      stream=None):
    """out[s, h] = softmax(scale * q[s, h] K^T) V over the paged cache of sequence s.

    q, out [S, Hq, d] (fp32 or bf16); k_cache/v_cache [NB, Hkv, B, d], B = 8, 16 or 32
    tokens per block (fp32, bf16, fp8-e4m3 as float8_e4m3fn/uint8, or int8);
    block_tables int32 [S, MB]; context_lens
    int32 [S]; k_scales/v_scales fp32 [NB, Hkv] for fp8 and int8; k_zeros/v_zeros int32
    [NB, Hkv] for int8; lse_out fp32 [S, Hq] or None; workspace a uint8 CUDA tensor of at
    least ``workspace_size(...)`` bytes when partition_size > 0.
    """
    torch = _torch()
    desc = decode_desc_for(q, k_cache, block_tables, partition_size)
    if tuple(v_cache.shape) != tuple(k_cache.shape) or v_cache.dtype != k_cache.dtype:
        raise ValueError("k_cache and v_cache differ")
    if tuple(out.shape) != tuple(q.shape) or out.dtype != q.dtype:
        raise ValueError("out must match q")
    if block_tables.shape[0] != q.shape[0] or tuple(context_lens.shape) != (q.shape[0],):
        raise ValueError("block_tables / context_lens do not match q")
    if lse_out is not None and tuple(lse_out.shape) != tuple(q.shape[:2]):
        raise ValueError("lse_out must be [S, Hq]")
    for sc in (k_scales, v_scales, k_zeros, v_zeros):
        if sc is not None and tuple(sc.shape) != tuple(k_cache.shape[:2]):
            raise ValueError("scales / zero points must be [num_blocks, num_kv_heads]")
    ws_need = workspace_size(desc, max_context_len)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.paged_attn_decode(
        _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), _dev(context_lens, "context_lens", torch.int32),
        ctypes.c_float(scale), _dev(out, "out"), ctypes.byref(desc), int(max_context_len),
        _dev(k_scales, "k_scales", torch.float32), _dev(v_scales, "v_scales", torch.float32),
        _dev(k_zeros, "k_zeros", torch.int32), _dev(v_zeros, "v_zeros", torch.int32),
        _dev(lse_out, "lse_out", torch.float32), _dev(workspace, "workspace"), ws_bytes,
        _stream(stream))
    if st == PA_ERR_WORKSPACE:
        raise PagedAttnError(st, f"paged_attn_decode needs {ws_need} workspace bytes")
    _check(st, "paged_attn_decode")
    return out


def paged_attn_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start,
                       scale: float, out, *, max_query_len: int, max_context_len: int,
                       k_scales=None, v_scales=None, k_zeros=None, v_zeros=None, lse_out=None,
                       stream=None):
    """Causal attention of a step's new tokens over the paged cache.

    q, out [T, Hq, d]: the new tokens of every sequence, sequence s owning rows
    query_start[s] .. query_start[s+1]-1 (query_start int32 [S+1]); their K/V must already
    be in the cache as the last tokens of context_lens[s]. Row i of sequence s attends to
    positions 0 .. context_lens[s] - n_s + i. Other arguments as in paged_attn_decode.
    """
    torch = _torch()
    T, Hq, d = q.shape
    NB, Hkv, B, d2 = k_cache.shape
    if d2 != d:
        raise ValueError("head_dim of q and cache differ")
    S = block_tables.shape[0]
    if tuple(context_lens.shape) != (S,) or tuple(query_start.shape) != (S + 1,):
        raise ValueError("context_lens must be [S] and query_start [S + 1]")
    if tuple(v_cache.shape) != tuple(k_cache.shape) or v_cache.dtype != k_cache.dtype:
        raise ValueError("k_cache and v_cache differ")
    if tuple(out.shape) != tuple(q.shape) or out.dtype != q.dtype:
        raise ValueError("out must match q")
    if lse_out is not None and tuple(lse_out.shape) != (T, Hq):
        raise ValueError("lse_out must be [T, Hq]")
    for sc in (k_scales, v_scales, k_zeros, v_zeros):
        if sc is not None and tuple(sc.shape) != tuple(k_cache.shape[:2]):
            raise ValueError("scales / zero points must be [num_blocks, num_kv_heads]")
    qd = _dtype_code(q.dtype)
    desc = make_desc(S, Hq, Hkv, d, block_tables.shape[1], NB, 0, qd, _dtype_code(k_cache.dtype),
                     qd, block_size=B)
    st = _lib.paged_attn_prefill(
        _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32),
        _dev(query_start, "query_start", torch.int32), int(T), int(max_query_len),
        ctypes.c_float(scale), _dev(out, "out"), ctypes.byref(desc), int(max_context_len),
        _dev(k_scales, "k_scales", torch.float32), _dev(v_scales, "v_scales", torch.float32),
        _dev(k_zeros, "k_zeros", torch.int32), _dev(v_zeros, "v_zeros", torch.int32),
        _dev(lse_out, "lse_out", torch.float32), _stream(stream))
    _check(st, "paged_attn_prefill")
    return out


NOALLOC_SCRATCH_BYTES = 32 << 20


def paged_attn_decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                              out, *, max_context_len: int, partition_size: int = 0,
                              k_scales=None, v_scales=None, k_zeros=None, v_zeros=None,
                              lse_out=None, stream=None):
    """paged_attn_decode without a caller workspace: the split-KV scratch comes from a fixed
    array inside the library (at most NOALLOC_SCRATCH_BYTES per GPU), for callers that
    cannot allocate device memory. Overlapping calls on one GPU race on that array."""
    torch = _torch()
    desc = decode_desc_for(q, k_cache, block_tables, partition_size)
    if tuple(out.shape) != tuple(q.shape) or out.dtype != q.dtype:
        raise ValueError("out must match q")
    st = _lib.paged_attn_decode_noalloc(
        _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), _dev(context_lens, "context_lens", torch.int32),
        ctypes.c_float(scale), _dev(out, "out"), ctypes.byref(desc), int(max_context_len),
        _dev(k_scales, "k_scales", torch.float32), _dev(v_scales, "v_scales", torch.float32),
        _dev(k_zeros, "k_zeros", torch.int32), _dev(v_zeros, "v_zeros", torch.int32),
        _dev(lse_out, "lse_out", torch.float32), _stream(stream))
    _check(st, "paged_attn_decode_noalloc")
    return out


def reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, *, k_scales=None, v_scales=None,
                      k_zeros=None, v_zeros=None, stream=None):
    """Writes k, v [T, Hkv, d] (rows may be strided along T) into the cache slots given by
    slot_mapping int64 [T] (negative = skip); fp8 / int8 caches take the per-(block, kv
    head) scales (and int8 zero points) of the destination blocks."""
    torch = _torch()
    T, Hkv, d = k.shape
    NB, Hkv2, B, d2 = k_cache.shape
    if (Hkv, d) != (Hkv2, d2) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k/v shape does not match the cache")
    if tuple(slot_mapping.shape) != (T,):
        raise ValueError("slot_mapping must be [T]")
    for x, n in ((k, "k"), (v, "v")):
        if x.stride(2) != 1 or x.stride(1) != d:
            raise ValueError(f"{n} rows must be contiguous [Hkv, d]")
    for c, n in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        if not c.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    st = _lib.reshape_and_cache(
        _dev(k, "k", contiguous=False), _dev(v, "v", contiguous=False), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache"), _dev(slot_mapping, "slot_mapping", torch.int64), T,
        int(k.stride(0)), int(v.stride(0)), Hkv, d, B, NB, _dtype_code(k.dtype),
        _dtype_code(k_cache.dtype), _dev(k_scales, "k_scales", torch.float32),
        _dev(v_scales, "v_scales", torch.float32), _dev(k_zeros, "k_zeros", torch.int32),
        _dev(v_zeros, "v_zeros", torch.int32), _stream(stream))
    _check(st, "reshape_and_cache")


def copy_blocks(k_cache, v_cache, pairs, *, k_scales=None, v_scales=None, k_zeros=None,
                v_zeros=None, stream=None):
    """Copies whole blocks (K, V and the quantisation scales / zero points) for every
    (src, dst) row of pairs int32 [n, 2]."""
    torch = _torch()
    NB, Hkv, B, d = k_cache.shape
    if pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be [n, 2]")
    st = _lib.copy_blocks(
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), _dev(k_scales, "k_scales", torch.float32),
        _dev(v_scales, "v_scales", torch.float32), _dev(k_zeros, "k_zeros", torch.int32),
        _dev(v_zeros, "v_zeros", torch.int32), _dev(pairs, "pairs", torch.int32),
        int(pairs.shape[0]), Hkv, d, B, NB, _dtype_code(k_cache.dtype), _stream(stream))
    _check(st, "copy_blocks")


def device_error(stream=None) -> int:
    """Reads and clears the device error word (bits PA_DEVERR_*); synchronises the stream."""
    bits = ctypes.c_int(0)
    st = _lib.pa_device_error(ctypes.byref(bits), _stream(stream))
    if st not in (PA_OK, PA_ERR_DEVICE):
        _check(st, "pa_device_error")
    return bits.value


def sha256(data: bytes) -> bytes:
    """SHA-256 computed by the library (the hash its prefix cache chains)."""
    buf = (ctypes.c_uint8 * 32)()
    b = bytes(data)
    _lib.pa_sha256(ctypes.c_char_p(b), len(b), buf)
    return bytes(buf)


class BlockAllocator:
    """Host block allocator (FIFO free queue, ref_count, fork, append with copy-on-write)."""

    def __init__(self, num_blocks: int, block_size: int = 16, order: Optional[Sequence[int]] = None):
        if order is None:
            self._h = _lib.pa_alloc_create(num_blocks, block_size)
        else:
            arr = np.ascontiguousarray(order, dtype=np.int32)
            if arr.shape != (num_blocks,):
                raise ValueError("order must have num_blocks entries")
            self._h = _lib.pa_alloc_create_ordered(num_blocks, block_size,
                                                   arr.ctypes.data_as(ctypes.c_void_p))
        if not self._h:
            raise ValueError("pa_alloc_create failed (bad sizes or order)")
        self.num_blocks = num_blocks
        self.block_size = block_size

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _lib is not None:  # module globals may already be gone at interpreter exit
            _lib.pa_alloc_destroy(h)
            self._h = None

    def num_free(self) -> int:
        return _lib.pa_alloc_num_free(self._h)

    def ref_count(self, block: int) -> int:
        return _lib.pa_alloc_ref_count(self._h, int(block))

    def add_seq(self, seq: int, num_tokens: int) -> np.ndarray:
        slots = np.empty(max(num_tokens, 0), dtype=np.int64)
        _check(_lib.pa_alloc_add_seq(self._h, int(seq), int(num_tokens),
                                     slots.ctypes.data_as(ctypes.c_void_p)), "pa_alloc_add_seq")
        return slots

    def add_seq_tokens(self, seq: int, tokens) -> Tuple[np.ndarray, int]:
        """New sequence with token ids (prefix caching): returns (slots, cached_tokens)."""
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        slots = np.empty(tok.size, dtype=np.int64)
        cached = ctypes.c_int(0)
        _check(_lib.pa_alloc_add_seq_tokens(self._h, int(seq), tok.ctypes.data_as(ctypes.c_void_p),
                                            int(tok.size), slots.ctypes.data_as(ctypes.c_void_p),
                                            ctypes.byref(cached)), "pa_alloc_add_seq_tokens")
        return slots, cached.value

    def num_cached(self) -> int:
        return _lib.pa_alloc_num_cached(self._h)

    def cache_stats(self) -> Tuple[int, int]:
        """(blocks reused by hits, cache entries evicted) since creation."""
        h, e = ctypes.c_int64(0), ctypes.c_int64(0)
        _check(_lib.pa_alloc_cache_stats(self._h, ctypes.byref(h), ctypes.byref(e)),
               "pa_alloc_cache_stats")
        return h.value, e.value

    def block_hash(self, block: int) -> Optional[bytes]:
        buf = (ctypes.c_uint8 * 32)()
        if not _lib.pa_alloc_block_hash(self._h, int(block), buf):
            return None
        return bytes(buf)

    def fork(self, parent: int, child: int) -> None:
        _check(_lib.pa_alloc_fork(self._h, int(parent), int(child)), "pa_alloc_fork")

    def append(self, seq: int, num_tokens: int) -> Tuple[np.ndarray, list]:
        slots = np.empty(max(num_tokens, 0), dtype=np.int64)
        pair = np.empty(2, dtype=np.int32)
        n = ctypes.c_int(0)
        _check(_lib.pa_alloc_append(self._h, int(seq), int(num_tokens),
                                    slots.ctypes.data_as(ctypes.c_void_p),
                                    pair.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n)),
               "pa_alloc_append")
        return slots, ([(int(pair[0]), int(pair[1]))] if n.value else [])

    def append_batch(self, seqs, num_tokens) -> Tuple[np.ndarray, np.ndarray]:
        """Appends num_tokens[i] tokens to seqs[i] for every i in one library call, in order,
        all or nothing (``NoBlocks`` and no change when the whole batch does not fit).
        ``num_tokens`` may be one int for every sequence. Returns (slots of all the tokens,
        sequence after sequence; int32 [k, 2] copy-on-write pairs in batch order)."""
        ids = np.ascontiguousarray(seqs, dtype=np.int32).ravel()
        cnt = np.ascontiguousarray(np.broadcast_to(np.asarray(num_tokens, dtype=np.int32),
                                                   ids.shape), dtype=np.int32)
        slots = np.empty(int(cnt.sum()) if cnt.size else 0, dtype=np.int64)
        pairs = np.empty((max(ids.size, 1), 2), dtype=np.int32)
        n = ctypes.c_int(0)
        _check(_lib.pa_alloc_append_batch(self._h, int(ids.size),
                                          ids.ctypes.data_as(ctypes.c_void_p),
                                          cnt.ctypes.data_as(ctypes.c_void_p),
                                          slots.ctypes.data_as(ctypes.c_void_p),
                                          pairs.ctypes.data_as(ctypes.c_void_p),
                                          ctypes.byref(n)), "pa_alloc_append_batch")
        return slots, pairs[:n.value].copy()

    def free_seq(self, seq: int) -> None:
        _check(_lib.pa_alloc_free_seq(self._h, int(seq)), "pa_alloc_free_seq")

    def block_table(self, seq: int) -> list:
        n = _lib.pa_alloc_block_table(self._h, int(seq), None, 0)
        if n < 0:
            raise PagedAttnError(PA_ERR_INVALID, "pa_alloc_block_table")
        out = np.empty(n, dtype=np.int32)
        _lib.pa_alloc_block_table(self._h, int(seq), out.ctypes.data_as(ctypes.c_void_p), n)
        return out.tolist()

    def seq_len(self, seq: int) -> int:
        return _lib.pa_alloc_seq_len(self._h, int(seq))

    def free_queue(self) -> list:
        n = _lib.pa_alloc_free_queue(self._h, None, 0)
        out = np.empty(n, dtype=np.int32)
        _lib.pa_alloc_free_queue(self._h, out.ctypes.data_as(ctypes.c_void_p), n)
        return out.tolist()

    def padded_tables(self, seqs: Sequence[int], max_blocks: int) -> np.ndarray:
        out = np.full((len(seqs), max_blocks), -1, dtype=np.int32)
        for i, s in enumerate(seqs):
            n = _lib.pa_alloc_block_table(self._h, int(s),
                                          out[i].ctypes.data_as(ctypes.c_void_p), max_blocks)
            if n < 0 or n > max_blocks:
                raise PagedAttnError(PA_ERR_INVALID, "block table wider than max_blocks")
        return out
