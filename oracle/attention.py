"""Decode and prefill attention over the paged cache, float64 (test infrastructure only).

[KVPaged] "Core principle: what is the KV cache": attention(Q, K, V) = softmax(Q K^T /
sqrt(d_k)) V; at decode one new query attends to the cached keys and values of all earlier
tokens. [Ch4PA] "PagedAttention algorithm": given the query and the block table, the kernel
looks each logical block up and gathers the non-contiguous K and V blocks before computing
attention. [KVPaged] "GQA and MQA": query heads are grouped and every group shares one KV
head (read: contiguous groups, query head h uses kv head h // (Hq / Hkv)).

The oracle is the plain definition: gather through the block table into contiguous arrays,
decode every stored element exactly to float64 (fp8: E4M3 value * the block's scale; int8:
(code - zero point) * scale), then
z = scale * q . K_t, p = exp(z - max z) / sum exp(z - max z), out = sum_t p_t V_t and
lse = max z + log sum exp(z - max z). ``context_lens[s]`` counts the token being decoded.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Tuple

import numpy as np

from .codecs import bf16_decode, e4m3_decode


def decode_values(codes: np.ndarray, dtype: str) -> np.ndarray:
    """Storage codes -> float64 values (exact)."""
    if dtype == "f32":
        return np.asarray(codes, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return bf16_decode(codes)
    if dtype == "fp8":
        return e4m3_decode(codes)
    raise ValueError(dtype)


def gather_kv(k_cache, v_cache, block_row, ctx: int, kvh: int, kv_dtype: str,
              k_scales=None, v_scales=None, k_zeros=None,
              v_zeros=None) -> Tuple[np.ndarray, np.ndarray]:
    """Contiguous float64 K and V [ctx, d] of one (sequence, kv head), read through the
    block table row: token t lives in physical block block_row[t // B] at offset t % B.
    fp8: E4M3 value * scale; int8: (code - zero) * scale, of the token's block."""
    B = k_cache.shape[2]
    t = np.arange(ctx)
    blk = np.asarray(block_row, dtype=np.int64)[t // B]
    off = t % B
    if kv_dtype == "int8":
        K = k_cache[blk, kvh, off, :].astype(np.float64) - \
            np.asarray(k_zeros, dtype=np.float64)[blk, kvh][:, None]
        V = v_cache[blk, kvh, off, :].astype(np.float64) - \
            np.asarray(v_zeros, dtype=np.float64)[blk, kvh][:, None]
    else:
        K = decode_values(k_cache[blk, kvh, off, :], kv_dtype)
        V = decode_values(v_cache[blk, kvh, off, :], kv_dtype)
    if kv_dtype in ("fp8", "int8"):
        K = K * np.asarray(k_scales, dtype=np.float64)[blk, kvh][:, None]
        V = V * np.asarray(v_scales, dtype=np.float64)[blk, kvh][:, None]
    return K, V


def ref_decode(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
               block_tables: np.ndarray, context_lens: np.ndarray, scale: float,
               num_kv_heads: int, q_dtype: str, kv_dtype: str,
               k_scales: Optional[np.ndarray] = None, v_scales: Optional[np.ndarray] = None,
               seqs: Optional[Iterable[int]] = None, k_zeros: Optional[np.ndarray] = None,
               v_zeros: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """out [S, Hq, d] and lse [S, Hq] in float64 for the sequences in ``seqs`` (default all;
    rows of other sequences are NaN). ctx = 0 gives out = 0 and lse = -inf."""
    S, Hq, d = q.shape
    G = Hq // num_kv_heads
    qv = decode_values(q, q_dtype)
    out = np.full((S, Hq, d), np.nan)
    lse = np.full((S, Hq), np.nan)
    for s in (range(S) if seqs is None else seqs):
        ctx = int(context_lens[s])
        for kvh in range(num_kv_heads):
            hs = slice(kvh * G, (kvh + 1) * G)
            if ctx == 0:
                out[s, hs] = 0.0
                lse[s, hs] = -np.inf
                continue
            K, V = gather_kv(k_cache, v_cache, block_tables[s], ctx, kvh, kv_dtype,
                             k_scales, v_scales, k_zeros, v_zeros)
            z = scale * (qv[s, hs] @ K.T)          # [G, ctx]
            m = z.max(axis=1, keepdims=True)
            e = np.exp(z - m)
            l = e.sum(axis=1, keepdims=True)
            out[s, hs] = (e @ V) / l
            lse[s, hs] = (m + np.log(l))[:, 0]
    return out, lse


def brute_force_attention(q_vec, keys, values, scale: float):
    """Textbook single-query attention with Python loops and ``math.exp`` on contiguous
    lists: out_j = sum_t w_t V[t][j], w_t = exp(s_t) / sum_u exp(s_u), s_t = scale q.K[t].
    Deliberately written without the max shift, for small well-scaled inputs only."""
    s = [scale * sum(float(a) * float(b) for a, b in zip(q_vec, k)) for k in keys]
    w = [math.exp(x) for x in s]
    tot = sum(w)
    d = len(values[0])
    return [sum(w[t] * float(values[t][j]) for t in range(len(keys))) / tot for j in range(d)], \
        math.log(tot)


def ref_prefill(q: np.ndarray, query_start: np.ndarray, k_cache: np.ndarray,
                v_cache: np.ndarray, block_tables: np.ndarray, context_lens: np.ndarray,
                scale: float, num_kv_heads: int, q_dtype: str, kv_dtype: str,
                k_scales: Optional[np.ndarray] = None, v_scales: Optional[np.ndarray] = None,
                k_zeros: Optional[np.ndarray] = None, v_zeros: Optional[np.ndarray] = None,
                seqs: Optional[Iterable[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Causal attention of a step's new tokens over the paged cache (prefill).

    [KVPaged] "Core principle: what is the KV cache": the prompt's K and V are computed
    once and cached, each token attending to itself and every earlier token; "Prefix
    sharing and copy-on-write": a shared prefix's KV is computed once, so a step may bring
    only the tokens after a cached prefix. Reading: sequence s brings
    n_s = query_start[s+1] - query_start[s] new tokens (rows query_start[s].. of q
    [T, Hq, d]) whose K/V were written into the cache first, as the last n_s of its
    context_lens[s] positions. Row i of the sequence sits at position
    p = context_lens[s] - n_s + i and attends to positions 0..p through the block table:
    z_t = scale * q . K_t for t <= p, out = sum_t softmax(z)_t V_t, lse = log sum_t e^z_t.
    Returns out [T, Hq, d] and lse [T, Hq] in float64; rows of sequences outside ``seqs``
    are NaN.
    """
    T, Hq, d = q.shape
    G = Hq // num_kv_heads
    qv = decode_values(q, q_dtype)
    out = np.full((T, Hq, d), np.nan)
    lse = np.full((T, Hq), np.nan)
    S = len(context_lens)
    for s in (range(S) if seqs is None else seqs):
        r0, r1 = int(query_start[s]), int(query_start[s + 1])
        n, ctx = r1 - r0, int(context_lens[s])
        if n == 0:
            continue
        assert 0 < n <= ctx
        pos = ctx - n + np.arange(n)                       # position of each new token
        allowed = np.arange(ctx)[None, :] <= pos[:, None]  # [n, ctx]
        for kvh in range(num_kv_heads):
            K, V = gather_kv(k_cache, v_cache, block_tables[s], ctx, kvh, kv_dtype,
                             k_scales, v_scales, k_zeros, v_zeros)
            for g in range(G):
                h = kvh * G + g
                z = scale * (qv[r0:r1, h] @ K.T)            # [n, ctx]
                z = np.where(allowed, z, -np.inf)
                m = z.max(axis=1, keepdims=True)
                e = np.exp(z - m)
                l = e.sum(axis=1, keepdims=True)
                out[r0:r1, h] = (e @ V) / l
                lse[r0:r1, h] = (m + np.log(l))[:, 0]
    return out, lse
