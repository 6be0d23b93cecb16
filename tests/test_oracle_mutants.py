"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of ``oracle/`` (a dropped term, a wrong sign, index
or rounding rule, a transposed operand, a missed reference count), runs the CPU pins of the
oracle against that copy in a separate interpreter, and expects at least one of them to
fail. The unchanged copy must pass. A planted mistake that no pin catches marks a pin that
is missing.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PIN_FILES = ["test_oracle_codecs.py", "test_oracle_facts.py", "test_oracle_paged.py",
             "test_oracle_attention.py", "test_oracle_prefill.py",
             "test_oracle_hashes.py", "test_workloads_prefill.py", "test_workloads_decode.py"]

# id -> (file under oracle/, text, replacement). The text must occur exactly once.
MUTANTS = {
    # attention
    "score_scale_dropped": ("attention.py", "z = scale * (qv[s, hs] @ K.T)", "z = (qv[s, hs] @ K.T)"),
    "lse_without_max": ("attention.py", "lse[s, hs] = (m + np.log(l))[:, 0]",
                        "lse[s, hs] = np.log(l)[:, 0]"),
    "gqa_interleaved": ("attention.py", "hs = slice(kvh * G, (kvh + 1) * G)",
                        "hs = slice(kvh, Hq, num_kv_heads)"),
    "offset_reversed_in_block": ("attention.py", "off = t % B", "off = B - 1 - t % B"),
    "last_token_dropped": ("attention.py", "        ctx = int(context_lens[s])\n",
                           "        ctx = max(int(context_lens[s]) - 1, 1)\n"),
    "fp8_v_scale_dropped": ("attention.py",
                            "V = V * np.asarray(v_scales, dtype=np.float64)[blk, kvh][:, None]",
                            "V = V"),
    "fp8_k_scale_dropped": ("attention.py",
                            "K = K * np.asarray(k_scales, dtype=np.float64)[blk, kvh][:, None]",
                            "K = K"),
    "int8_k_zero_added": ("attention.py", "K = k_cache[blk, kvh, off, :].astype(np.float64) - \\",
                          "K = k_cache[blk, kvh, off, :].astype(np.float64) + \\"),
    "int8_v_zero_added": ("attention.py", "V = v_cache[blk, kvh, off, :].astype(np.float64) - \\",
                          "V = v_cache[blk, kvh, off, :].astype(np.float64) + \\"),
    "int8_v_zero_from_k": ("attention.py",
                           "            np.asarray(v_zeros, dtype=np.float64)[blk, kvh][:, None]",
                           "            np.asarray(k_zeros, dtype=np.float64)[blk, kvh][:, None]"),
    "prefill_mask_strict": ("attention.py", "<= pos[:, None]", "< pos[:, None]"),
    "prefill_mask_open": ("attention.py", "z = np.where(allowed, z, -np.inf)", "pass"),
    "prefill_tokens_at_front": ("attention.py", "pos = ctx - n + np.arange(n)", "pos = np.arange(n)"),
    "prefill_head_interleaved": ("attention.py", "h = kvh * G + g", "h = g * num_kv_heads + kvh"),
    "prefill_lse_without_max": ("attention.py", "lse[r0:r1, h] = (m + np.log(l))[:, 0]",
                                "lse[r0:r1, h] = np.log(l)[:, 0]"),
    "prefill_scales_swapped": ("attention.py",
                               "k_scales, v_scales, k_zeros, v_zeros)\n            for g in",
                               "v_scales, k_scales, k_zeros, v_zeros)\n            for g in"),
    "prefill_zeros_swapped": ("attention.py",
                              "k_scales, v_scales, k_zeros, v_zeros)\n            for g in",
                              "k_scales, v_scales, v_zeros, k_zeros)\n            for g in"),
    "prefill_state_zeros_swapped": ("flows.py", "state.k_zeros, state.v_zeros, seqs=seqs)",
                                    "state.v_zeros, state.k_zeros, seqs=seqs)"),
    "state_tokens_shifted": ("flows.py", "ref_reshape_and_cache(k[:-1], v[:-1], kc, vc, pre[s],",
                             "ref_reshape_and_cache(k[1:], v[1:], kc, vc, pre[s],"),
    # codecs
    "e4m3_bias_8": ("codecs.py", "2.0 ** (e - 7)", "2.0 ** (e - 8)"),
    "e4m3_subnormal_exponent": ("codecs.py", "2.0 ** (1 - 7)", "2.0 ** (0 - 7)"),
    "e4m3_ties_to_odd": ("codecs.py", "((d_hi == d_lo) & ((hi & 1) == 0))",
                         "((d_hi == d_lo) & ((hi & 1) == 1))"),
    "e4m3_nan_code": ("codecs.py", "code[nan] = np.uint8(0x7F)", "code[nan] = np.uint8(0x7E)"),
    "bf16_ties_up": ("codecs.py", "up = (rem > 0x8000) |", "up = (rem >= 0x8000) |"),
    "bf16_truncates": ("codecs.py", "out = (lo + up.astype(np.uint64)).astype(np.uint16)",
                       "out = lo.astype(np.uint16)"),
    "int8_floor": ("codecs.py", "np.rint(y.astype(np.float64))", "np.floor(y.astype(np.float64))"),
    "int8_wraps": ("codecs.py", "np.clip(r, -128, 127).astype(np.int8)", "r.astype(np.int8)"),
    "int8_decode_zero_added": ("codecs.py", "astype(np.float64) - np.asarray(zero, dtype=np.float64)",
                               "astype(np.float64) + np.asarray(zero, dtype=np.float64)"),
    # allocator, slots, cache write, block copy
    "slot_block_offset_swapped": ("paged.py",
                                  "return int(block_table_row[pos // block_size]) * block_size"
                                  " + pos % block_size",
                                  "return int(block_table_row[pos % block_size]) * block_size"
                                  " + pos // block_size"),
    "free_queue_lifo": ("paged.py", "b = self.free.popleft()", "b = self.free.pop()"),
    "freed_block_to_front": ("paged.py", "self.free.append(b)", "self.free.appendleft(b)"),
    "fork_keeps_ref_counts": ("paged.py", "        for b in self.tables[child]:\n"
                              "            self.refs[b] += 1\n", ""),
    "cow_keeps_old_reference": ("paged.py", "            self.refs[old] -= 1\n", ""),
    "cow_of_full_block": ("paged.py", "cow = num_tokens > 0 and L % B != 0 and",
                          "cow = num_tokens > 0 and"),
    "cow_not_reported": ("paged.py", "            pairs.append((old, new))\n", ""),
    "grow_off_by_one": ("paged.py", "grow = -(-(L + num_tokens) // B) - -(-L // B)",
                        "grow = (L + num_tokens) // B - L // B"),
    "write_block_offset_swapped": ("paged.py", "blk, off = int(slot // B), int(slot % B)",
                                   "off, blk = int(slot // B) % B, int(slot % B)"),
    "write_padding_slot": ("paged.py", "        if slot < 0:\n            continue\n",
                           "        if slot < -1:\n            continue\n"),
    "write_v_into_k": ("paged.py", "for x, cache, sc, zp in ((k, k_cache, k_scales, k_zeros), "
                       "(v, v_cache, v_scales, v_zeros)):",
                       "for x, cache, sc, zp in ((k, k_cache, k_scales, k_zeros), "
                       "(k, v_cache, v_scales, v_zeros)):"),
    "fp8_write_multiplies": ("paged.py", "        y = (xf / scale[..., None].astype(np.float32))"
                             ".astype(np.float32)\n        return e4m3_encode(y)",
                             "        y = (xf * scale[..., None].astype(np.float32))"
                             ".astype(np.float32)\n        return e4m3_encode(y)"),
    "int8_write_without_zero": ("paged.py", "return int8_encode(y, np.asarray(zero)[..., None])",
                                "return int8_encode(y, 0)"),
    "copy_blocks_reversed": ("paged.py", "        k_cache[dst] = k_cache[src]\n"
                             "        v_cache[dst] = v_cache[src]\n",
                             "        k_cache[src] = k_cache[dst]\n"
                             "        v_cache[src] = v_cache[dst]\n"),
    "copy_blocks_without_scales": ("paged.py", "                arr[dst] = arr[src]\n",
                                   "                pass\n"),
    "batch_not_atomic": ("paged.py", "            self.__dict__.update(saved)\n", ""),
    "hash_not_chained": ("paged.py", "            m.update(parent)\n", "            pass\n"),
    "hash_big_endian": ("paged.py", 'dtype="<i4"', 'dtype=">i4"'),
    # closed forms
    "kv_bytes_without_factor_2": ("facts.py", "num_layers * 2 * batch", "num_layers * batch"),
    "blocks_floor": ("facts.py", "return -(-tokens // block_size)", "return tokens // block_size"),
    "sharing_savings_denominator": ("facts.py", "(R - 1) * prefix / (R * (prefix + suffix))",
                                    "(R - 1) * prefix / ((R - 1) * (prefix + suffix))"),
}


def _copy_tree(dst):
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__", "*.so", "*.o"))
    shutil.copytree(os.path.join(ROOT, "workloads"), os.path.join(dst, "workloads"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.makedirs(os.path.join(dst, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    for f in ["conftest.py"] + PIN_FILES:
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), os.path.join(dst, "pytest.ini"))


def _plant(dst, case):
    if case is None:
        return
    fname, old, new = MUTANTS[case]
    path = os.path.join(dst, "oracle", fname)
    with open(path) as f:
        src = f.read()
    assert src.count(old) == 1, f"{case}: the planted text occurs {src.count(old)} times"
    with open(path, "w") as f:
        f.write(src.replace(old, new))


# the pins closest to each oracle file run first, so that a caught mistake stops early
FIRST = {"attention.py": ["test_oracle_attention.py", "test_oracle_prefill.py"],
         "flows.py": ["test_workloads_decode.py", "test_oracle_prefill.py",
                      "test_oracle_attention.py"],
         "codecs.py": ["test_oracle_codecs.py"],
         "paged.py": ["test_oracle_paged.py", "test_oracle_hashes.py"],
         "facts.py": ["test_oracle_facts.py"]}


def _run_pins(dst, case):
    first = FIRST[MUTANTS[case][0]] if case else []
    files = first + [f for f in PIN_FILES if f not in first]
    env = {k: v for k, v in os.environ.items() if k != "PYTHONPATH"}
    env.update(PYTHONDONTWRITEBYTECODE="1", OMP_NUM_THREADS="1", MKL_NUM_THREADS="1",
               OPENBLAS_NUM_THREADS="1")
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu",
                        *[os.path.join("tests", f) for f in files]],
                       cwd=dst, env=env, capture_output=True, text=True, timeout=900)
    return p.returncode, p.stdout[-2000:] + p.stderr[-2000:]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    """Runs the pins on the unchanged copy and on every planted copy, a few at a time."""
    base = tmp_path_factory.mktemp("oracle_mutants")
    cases = [None] + list(MUTANTS)

    def one(case):
        dst = os.path.join(base, case or "unchanged")
        os.makedirs(dst)
        _copy_tree(dst)
        _plant(dst, case)
        return case, _run_pins(dst, case)

    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with cf.ThreadPoolExecutor(workers) as ex:
        return dict(ex.map(one, cases))


def test_unchanged_oracle_passes_its_pins(outcomes):
    rc, log = outcomes[None]
    assert rc == 0, log


@pytest.mark.parametrize("case", list(MUTANTS))
def test_planted_mistake_is_caught(outcomes, case):
    rc, log = outcomes[case]
    # 1: some pin failed. 0 would mean the mistake went unnoticed; anything else is a
    # broken harness (collection error, interpreter crash), not a caught mistake.
    assert rc == 1, f"planted '{case}' -> pytest exit {rc}\n{log}"
