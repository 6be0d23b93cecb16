"""A decode step of a synthetic workload, built on the GPU through the library.

Sets a workload up the way a serving step would see it — blocks allocated by the native
allocator in the draw's pool order, earlier tokens written into the pool with
reshape_and_cache — and exposes one decode step:

    copy_blocks(copy-on-write pairs)           (shared-prefix workload only)
    reshape_and_cache(this step's new K/V)
    paged_attn_decode(q) [+ log-sum-exp reduce when split into partitions]

K/V of the sequences in ``draw_seqs`` (default: all) comes from the seeded NumPy draw, so
an oracle can recompute exactly those sequences; every other sequence gets seeded N(0, 1)
values generated on the device (same distribution, same shapes), which keeps full-size
workloads quick to set up.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

from .cache import PagedKVCache


def _ceil_div(a, b):
    return -(-a // b)


class DeviceScenario:
    def __init__(self, draw, draw_seqs: Optional[Sequence[int]] = None, shared: bool = True,
                 partition_size: Optional[int] = None, device="cuda"):
        import torch
        self.torch = torch
        self.draw = draw
        wl = self.wl = draw.wl
        S, B, H, d = wl.num_seqs, wl.block_size, wl.num_kv_heads, wl.head_dim
        self.device = device
        self.draw_seqs = set(range(S)) if draw_seqs is None else set(draw_seqs)
        self.partition_size = wl.partition_size if partition_size is None else partition_size
        self.tdtype = torch.float32 if wl.in_dtype == "f32" else torch.bfloat16
        lens = draw.context_lens
        self.max_context_len = int(lens.max()) if S else 0
        self.max_blocks = max(1, _ceil_div(self.max_context_len, B))
        nb = wl.num_blocks
        self.is_shared = wl.shared_prefix is not None and shared
        if self.is_shared and wl.kv_dtype in ("fp8", "int8"):
            # per-block scales must be fixed before a block's first write; a shared partial
            # block is written before its copies exist, so the recipe has no single value
            raise NotImplementedError("quantised cache with a shared prefix")
        if wl.shared_prefix is not None and not shared:
            nb = max(nb, S * self.max_blocks)
        order = draw.pool_order if nb == wl.num_blocks else None
        self.cache = c = PagedKVCache(nb, H, d, wl.kv_dtype, B, device, order)

        # ---- allocation (host) ----
        pairs = []
        if self.is_shared:
            p, sfx = wl.shared_prefix
            pre_slots = {0: c.add_seq(0, p)}
            for ch in range(1, S):
                c.fork(0, ch)
            step_slots = {}
            for s in range(S):
                sl, pr = c.append(s, sfx)
                step_slots[s] = sl
                pairs += pr
            step_range = {s: (p, p + sfx) for s in range(S)}
            pre_range = {0: (0, p)}
        else:
            pre_slots, step_slots = {}, {}
            for s in range(S):
                pre_slots[s] = c.add_seq(s, int(lens[s]) - 1)
            for s in range(S):
                sl, pr = c.append(s, 1)
                assert not pr
                step_slots[s] = sl
            step_range = {s: (int(lens[s]) - 1, int(lens[s])) for s in range(S)}
            pre_range = {s: (0, int(lens[s]) - 1) for s in range(S)}
        self.cow_pairs = pairs
        self.block_tables = c.block_tables(range(S), self.max_blocks).to(device)
        self.context_lens = torch.from_numpy(lens.astype(np.int32)).to(device)
        tables_host = self.block_tables.cpu().numpy()

        # ---- K/V values and fp8 / int8 quantisation parameters (setup) ----
        step_k, step_v, step_sl = [], [], []
        for s in range(S):
            k, v = self._seq_kv(s)
            if wl.kv_dtype == "fp8":
                self._set_scales(s, k, v, tables_host[s])
            elif wl.kv_dtype == "int8":
                self._set_int8(s, k, v, tables_host[s])
            a, b = pre_range.get(s, (0, 0))
            if b > a:
                self._write(k[a:b], v[a:b], pre_slots[s])
            a, b = step_range[s]
            step_k.append(k[a:b])
            step_v.append(v[a:b])
            step_sl.append(step_slots[s])
        self.step_k = torch.cat(step_k).contiguous()
        self.step_v = torch.cat(step_v).contiguous()
        self.step_slots = torch.from_numpy(np.concatenate(step_sl).astype(np.int64)).to(device)
        self.pairs = (torch.tensor(pairs, dtype=torch.int32, device=device).reshape(-1, 2)
                      if pairs else None)

        # ---- decode inputs / outputs ----
        self.q = self._host_to_dev(draw.q)
        self.scale = float(np.float32(1.0 / math.sqrt(d)))
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty((S, wl.num_q_heads), dtype=torch.float32, device=device)
        nbytes = c.workspace_bytes(self.q, self.block_tables, self.max_context_len,
                                   self.partition_size)
        self.workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
        torch.cuda.synchronize()

    # -- helpers ------------------------------------------------------------------------------
    def _host_to_dev(self, x: np.ndarray):
        t = self.torch.from_numpy(np.ascontiguousarray(x))
        if self.wl.in_dtype == "bf16":
            t = t.view(self.torch.int16).view(self.torch.bfloat16)
        return t.to(self.device)

    def _seq_kv(self, s: int):
        torch = self.torch
        wl = self.wl
        if s in self.draw_seqs or (self.is_shared and s == 0):
            k, v = self.draw.kv(s)
            return self._host_to_dev(k), self._host_to_dev(v)
        n = int(self.draw.context_lens[s])
        g = torch.Generator(device=self.device)
        g.manual_seed(1_000_003 * (wl.seed + 1) + s)
        shape = (n, wl.num_kv_heads, wl.head_dim)
        k = torch.randn(shape, generator=g, device=self.device, dtype=torch.float32)
        v = torch.randn(shape, generator=g, device=self.device, dtype=torch.float32)
        return k.to(self.tdtype), v.to(self.tdtype)

    def _set_scales(self, s, k, v, table_row):
        """fp8 scales of sequence s: absmax/448 per (logical block, kv head) of the values
        it will hold (the workloads' recipe), placed at the block's physical index."""
        torch = self.torch
        wl = self.wl
        if s in self.draw_seqs or (self.is_shared and s == 0):
            lk, lv = self.draw.fp8_scales_logical(s)
            lk, lv = torch.from_numpy(lk).to(self.device), torch.from_numpy(lv).to(self.device)
        else:
            n, B = k.shape[0], wl.block_size
            nb = _ceil_div(n, B)
            res = []
            for x in (k, v):
                xf = x.float().abs()
                pad = nb * B - n
                if pad:
                    xf = torch.cat([xf, xf.new_zeros((pad,) + tuple(xf.shape[1:]))])
                am = xf.reshape(nb, B, wl.num_kv_heads, wl.head_dim).amax(dim=(1, 3))
                sc = am / 448.0
                sc[am == 0] = 1.0
                res.append(sc)
            lk, lv = res
        idx = torch.from_numpy(table_row[: lk.shape[0]].astype(np.int64)).to(self.device)
        self.cache.k_scales[idx] = lk
        self.cache.v_scales[idx] = lv

    def _set_int8(self, s, k, v, table_row):
        """int8 scale / zero point of sequence s per (logical block, kv head): min/max to the
        int8 range (the workloads' recipe), placed at the block's physical index."""
        torch = self.torch
        wl = self.wl
        if s in self.draw_seqs:
            lks, lkz, lvs, lvz = [torch.from_numpy(x).to(self.device)
                                  for x in self.draw.int8_params_logical(s)]
        else:
            n, B = k.shape[0], wl.block_size
            nb = _ceil_div(n, B)
            res = []
            for x in (k, v):
                xf = x.float()
                pad = nb * B - n
                if pad:  # pad with the block's first value so min/max cover valid tokens only
                    last = xf[(nb - 1) * B:(nb - 1) * B + 1].expand(pad, -1, -1)
                    xf = torch.cat([xf, last])
                xb = xf.reshape(nb, B, wl.num_kv_heads, wl.head_dim)
                mn = xb.amin(dim=(1, 3))
                mx = xb.amax(dim=(1, 3))
                sc = (mx - mn) / 255.0
                flat = mx <= mn
                sc = torch.where(flat, torch.ones_like(sc), sc)
                zp = torch.clamp(torch.round(-128.0 - mn / sc), -128, 127).to(torch.int32)
                zp = torch.where(flat, torch.zeros_like(zp), zp)
                res += [sc, zp]
            lks, lkz, lvs, lvz = res
        idx = torch.from_numpy(table_row[: lks.shape[0]].astype(np.int64)).to(self.device)
        c = self.cache
        c.k_scales[idx], c.k_zeros[idx], c.v_scales[idx], c.v_zeros[idx] = lks, lkz, lvs, lvz

    def _write(self, k, v, slots: np.ndarray):
        sl = self.torch.from_numpy(np.ascontiguousarray(slots, dtype=np.int64)).to(self.device)
        self.cache.write(k.contiguous(), v.contiguous(), sl)

    # -- the step --------------------------------------------------------------------------
    def step(self, stream=None):
        c = self.cache
        if self.pairs is not None:
            c.copy(self.pairs, stream=stream)
        c.write(self.step_k, self.step_v, self.step_slots, stream=stream)
        c.decode(self.q, self.block_tables, self.context_lens, self.scale, self.out,
                 max_context_len=self.max_context_len, partition_size=self.partition_size,
                 lse_out=self.lse, workspace=self.workspace, stream=stream)
        return self.out

    def resolved_partition(self) -> int:
        """The split partition the library takes for this step (0 = one pass)."""
        from . import decode_desc_for, partition_size_for
        return partition_size_for(decode_desc_for(self.q, self.cache.k_cache, self.block_tables,
                                                  self.partition_size), self.max_context_len)

    def launches_per_step(self) -> int:
        """The library's kernel launches in one step: block copies, cache write, decode."""
        from . import decode_desc_for, decode_launches
        desc = decode_desc_for(self.q, self.cache.k_cache, self.block_tables,
                               self.partition_size)
        return (1 if self.pairs is not None else 0) + 1 + decode_launches(
            desc, self.max_context_len)

    # -- algorithmic traffic of one step (bytes that must move) -----------------------------
    def kv_bytes(self) -> int:
        """K and V bytes decode must read: every cached token of every (seq, kv head)."""
        wl = self.wl
        es = {"f32": 4, "bf16": 2, "fp8": 1, "int8": 1}[wl.kv_dtype]
        return int(self.draw.context_lens.astype(np.int64).sum()) * 2 * wl.num_kv_heads * \
            wl.head_dim * es

    def step_bytes(self) -> dict:
        wl = self.wl
        S, Hq, Hkv, d, B = wl.num_seqs, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size
        es = {"f32": 4, "bf16": 2, "fp8": 1, "int8": 1}[wl.kv_dtype]
        ins = {"f32": 4, "bf16": 2}[wl.in_dtype]
        lens = self.draw.context_lens.astype(np.int64)
        blocks = int(np.sum(-(-lens // B)))
        kv = self.kv_bytes()
        scales = {"fp8": blocks * 2 * Hkv * 4, "int8": blocks * 2 * Hkv * 8}.get(wl.kv_dtype, 0)
        qo = S * Hq * d * ins * 2
        meta = blocks * 4 + S * 4
        decode = kv + scales + qo + meta
        T = int(self.step_k.shape[0])
        write = T * Hkv * d * (ins + es) * 2 + T * 8
        copy = len(self.cow_pairs) * 2 * Hkv * B * d * es * 2
        return {"decode": decode, "write": write, "copy": copy, "kv": kv,
                "total": decode + write + copy}


class PrefillScenario(DeviceScenario):
    """A prefill step of a synthetic workload, built on the GPU through the library.

    Blocks come from the native allocator in the draw's pool order: every sequence is added
    with its cached tokens (written beforehand with reshape_and_cache), then appends the
    step's new tokens. The step writes the new tokens' K/V and runs paged_attn_prefill for
    them. K/V of sequences outside ``draw_seqs`` is seeded N(0, 1) drawn on the device.
    """

    def __init__(self, draw, draw_seqs: Optional[Sequence[int]] = None, device="cuda"):
        import torch
        self.torch = torch
        self.draw = draw
        wl = self.wl = draw.wl
        S, B, H, d = wl.num_seqs, wl.block_size, wl.num_kv_heads, wl.head_dim
        self.device = device
        self.draw_seqs = set(range(S)) if draw_seqs is None else set(draw_seqs)
        self.is_shared = False
        self.partition_size = 0
        self.tdtype = torch.float32 if wl.in_dtype == "f32" else torch.bfloat16
        lens, qn = draw.context_lens, draw.query_lens
        self.max_context_len = int(lens.max()) if S else 0
        self.max_query_len = int(qn.max()) if S else 0
        self.max_blocks = max(1, _ceil_div(self.max_context_len, B))
        self.cache = c = PagedKVCache(wl.num_blocks, H, d, wl.kv_dtype, B, device,
                                      draw.pool_order)
        pre, new = {}, {}
        for s in range(S):
            pre[s] = c.add_seq(s, int(lens[s] - qn[s]))
        for s in range(S):
            sl, pr = c.append(s, int(qn[s]))
            assert not pr
            new[s] = sl
        self.cow_pairs, self.pairs = [], None
        self.block_tables = c.block_tables(range(S), self.max_blocks).to(device)
        self.context_lens = torch.from_numpy(lens.astype(np.int32)).to(device)
        self.query_start = torch.from_numpy(draw.query_start.astype(np.int32)).to(device)
        tables_host = self.block_tables.cpu().numpy()
        step_k, step_v, step_sl = [], [], []
        for s in range(S):
            k, v = self._seq_kv(s)
            if wl.kv_dtype == "fp8":
                self._set_scales(s, k, v, tables_host[s])
            elif wl.kv_dtype == "int8":
                self._set_int8(s, k, v, tables_host[s])
            cached = int(lens[s] - qn[s])
            if cached:
                self._write(k[:cached], v[:cached], pre[s])
            step_k.append(k[cached:])
            step_v.append(v[cached:])
            step_sl.append(new[s])
        self.step_k = torch.cat(step_k).contiguous()
        self.step_v = torch.cat(step_v).contiguous()
        self.step_slots = torch.from_numpy(np.concatenate(step_sl).astype(np.int64)).to(device)
        self.q = self._host_to_dev(draw.q)
        self.scale = float(np.float32(1.0 / math.sqrt(d)))
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty((self.q.shape[0], wl.num_q_heads), dtype=torch.float32,
                               device=device)
        self.workspace = None
        torch.cuda.synchronize()

    def step(self, stream=None):
        c = self.cache
        c.write(self.step_k, self.step_v, self.step_slots, stream=stream)
        c.prefill(self.q, self.block_tables, self.context_lens, self.query_start, self.scale,
                  self.out, max_query_len=self.max_query_len,
                  max_context_len=self.max_context_len, lse_out=self.lse, stream=stream)
        return self.out

    def launches_per_step(self) -> int:
        return 2

    def flops(self) -> int:
        """Multiply-adds x 2 of the causal products: every new token's row of S = q K^T
        and of P V over its visible keys (position + 1), for every query head."""
        wl = self.wl
        lens = self.draw.context_lens.astype(np.int64)
        qn = self.draw.query_lens.astype(np.int64)
        # sum over new tokens of (position + 1) = sum_{i<n} (ctx - n + i + 1)
        keys = int(np.sum(qn * (lens - qn) + qn * (qn + 1) // 2))
        return 4 * wl.head_dim * wl.num_q_heads * keys

