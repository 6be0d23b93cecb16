"""CPU oracle for the paged decode-attention hot path — TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct NumPy (float64 where floating point is involved). Only the
tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import it; the
product package never does, and this package imports nothing from the product. The two
share no code: only the seeded input generators in ``workloads`` serve both.

Modules
-------
codecs     bf16 and OCP FP8 E4M3 encode/decode, written from the format definitions.
facts      The pages' closed-form sizes: KV bytes, blocks per sequence, waste and sharing
           ratios, block-table overhead.
paged      Slot mapping, the reference block allocator (free queue, ref_count, fork,
           append with copy-on-write), the slot-mapped cache write and the block copy.
attention  Decode attention: gather each sequence's K/V through its block table into
           contiguous arrays, then softmax(q K^T * scale) V in float64.

Sources are cited as page title + section of the four pages on KV caches and PagedAttention:
  [KVFail]   "Transformer inference KV-cache memory-management failure modes"
             (knowledge.openakashic.com note)
  [OpsVLLM]  "How does vLLM PagedAttention manage the KV cache: throughput, latency, OOM"
             (opsoai.com)
  [KVPaged]  "KV cache and paged attention" (youngju.dev)
  [Ch4PA]    "Why PagedAttention cuts GPU memory waste by up to 95%" (iq-universe.github.io,
             ch4-paged-attention)

Parity status: every function here is pinned by a CPU test against printed values, closed
forms, invariants or brute force (``tests/test_oracle_*.py``); none is "parity unpinned".
The exact float bits of the GPU's attention output are covered by tolerances only.
"""
from . import codecs, facts, paged, attention  # noqa: F401
