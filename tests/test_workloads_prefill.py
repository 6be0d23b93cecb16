"""The prefill input recipe: seeded and reproducible, query ranges consistent with the
lengths (new tokens are the last ones of each context, never more than it), chunk and
whole-prompt forms, and the oracle's prefill state laid out as the allocator would."""
import numpy as np

import workloads
from oracle import flows


def test_draws_are_reproducible_and_consistent():
    for name, wl in workloads.PREFILL_WORKLOADS.items():
        if wl.num_seqs * 4096 > 200_000:
            wl = wl.scaled(num_seqs=3)
        d1, d2 = workloads.draw_prefill(wl), workloads.draw_prefill(wl)
        assert np.array_equal(d1.context_lens, d2.context_lens)
        assert np.array_equal(d1.q, d2.q)
        assert np.array_equal(d1.kv(0)[0], d2.kv(0)[0])
        qs = d1.query_start
        assert qs[0] == 0 and np.all(np.diff(qs) >= 0) and qs[-1] == d1.num_tokens
        assert np.array_equal(np.diff(qs), d1.query_lens)
        assert np.all(d1.query_lens <= d1.context_lens)
        assert d1.q.shape == (d1.num_tokens, wl.num_q_heads, wl.head_dim)
        assert d1.kv(0)[0].shape == (int(d1.context_lens[0]), wl.num_kv_heads, wl.head_dim)


def test_new_token_forms():
    base = workloads.PREFILL_WORKLOADS["chunked"].scaled(num_seqs=4, lens=("fixed", [3, 512, 600, 5000]),
                                                         num_blocks=1024)
    whole = workloads.draw_prefill(base.scaled(new=("full",)))
    assert np.array_equal(whole.query_lens, whole.context_lens)
    chunk = workloads.draw_prefill(base.scaled(new=("chunk", 512)))
    assert chunk.query_lens.tolist() == [3, 512, 512, 512]
    ragged = workloads.draw_prefill(base.scaled(new=("uniform", 0, 100)))
    assert np.all((ragged.query_lens >= 0) & (ragged.query_lens <= np.minimum(100, ragged.context_lens)))


def test_prefill_state_layout():
    d = workloads.draw_prefill("prefill_tiny")
    st = flows.build_prefill_state(d)
    B = d.wl.block_size
    for s in range(d.wl.num_seqs):
        n_blocks = -(-int(d.context_lens[s]) // B)
        row = st.block_tables[s]
        assert np.all(row[:n_blocks] >= 0) and np.all(row[n_blocks:] == -1)
        # the step's new tokens sit at the last positions, after the cached ones
        slots = st.step_slots[s]
        cached = int(d.context_lens[s] - d.query_lens[s])
        pos = np.arange(cached, int(d.context_lens[s]))
        assert np.array_equal(slots, row[pos // B] * B + pos % B)
