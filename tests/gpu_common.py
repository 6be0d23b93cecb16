"""Helpers shared by the GPU parity tests: tolerances and comparisons against the oracle."""
import numpy as np

# Tolerances of the decode output against the float64 oracle, per KV storage type:
# max-abs error (the stated bar) plus a relative-L2 bound per (seq, head) and an lse bound,
# which together catch a dropped partition that max-abs alone would miss at long contexts.
TOL = {
    "f32": dict(max_abs=1e-4, rel_l2=1e-5, lse=1e-3),
    "bf16": dict(max_abs=2e-2, rel_l2=1e-2, lse=1e-3),
    "fp8": dict(max_abs=3e-2, rel_l2=3e-2, lse=1e-3),
    "int8": dict(max_abs=3e-2, rel_l2=3e-2, lse=1e-3),
}


def to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def compare_decode(out_gpu, lse_gpu, out_ref, lse_ref, kv_dtype, seqs=None):
    """Returns a dict of error statistics and asserts the tolerances of ``kv_dtype``."""
    tol = TOL[kv_dtype]
    o = to_f64(out_gpu)
    l = to_f64(lse_gpu)
    if seqs is not None:
        o, l, out_ref, lse_ref = o[seqs], l[seqs], out_ref[seqs], lse_ref[seqs]
    err = np.abs(o - out_ref)
    max_abs = float(err.max()) if err.size else 0.0
    num = np.sqrt((err ** 2).sum(-1))
    den = np.sqrt((out_ref ** 2).sum(-1))
    rel = num / np.maximum(den, 1e-30)
    rel_l2 = float(rel.max()) if rel.size else 0.0
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(l), fin)
    lse_err = float(np.abs(l[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    stats = dict(max_abs=max_abs, rel_l2=rel_l2, lse=lse_err)
    assert max_abs <= tol["max_abs"], stats
    assert rel_l2 <= tol["rel_l2"], stats
    assert lse_err <= tol["lse"], stats
    return stats


def cache_codes(t) -> np.ndarray:
    """Device cache -> numpy array of its storage codes (float32 / uint16 / uint8)."""
    import torch
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
