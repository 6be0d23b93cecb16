"""Storage-format codecs of the oracle (test infrastructure only).

bfloat16: IEEE-754 binary32 with the low 16 bits dropped (1 sign, 8 exponent, 7 fraction
bits). Encoding from float32 rounds to nearest, ties to even, as the format is defined.

FP8 E4M3 (OCP 8-bit floating point specification, E4M3 variant): 1 sign bit, 4 exponent
bits with bias 7, 3 mantissa bits; no infinities; the only NaN patterns are S.1111.111; the
largest finite magnitude is 1.75 * 2^8 = 448; subnormals (exponent field 0) are
m/8 * 2^-6. The pages only say that FP8 stores one byte per element ([KVPaged], section
"KV quantization: FP8 and INT8"); the E4M3 layout is the one the fp8 KV cache here uses.

Encoding to E4M3 rounds to nearest, ties to even, and saturates finite values beyond 448 to
+-448 ("satfinite"); NaN encodes to 0x7F. It is written as a search over the 127 finite
magnitudes, so that it follows the definition rather than any bit trick.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_encode(x: np.ndarray) -> np.ndarray:
    """float32 -> uint16 bf16 bits, round to nearest even. Exact for the rounding step:
    the candidate values are the two bf16 neighbours of x; the nearer one wins, the one with
    an even last fraction bit on a tie."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lo = (u >> 16).astype(np.uint64)             # truncation (toward zero in magnitude)
    rem = u & 0xFFFF                              # dropped bits
    up = (rem > 0x8000) | ((rem == 0x8000) & ((lo & 1) == 1))
    out = (lo + up.astype(np.uint64)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def _e4m3_value(code: int) -> float:
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** (1 - 7)
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
_POS = E4M3_TABLE[:127]  # codes 0x00..0x7E: the finite non-negative magnitudes, increasing


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 E4M3 codes -> float64 (exact; NaN for S.1111.111)."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """float32 -> uint8 E4M3 codes: round to nearest, ties to even, saturate to +-448."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    a = np.abs(y.astype(np.float64))
    neg = np.signbit(y)
    # index of the first magnitude >= a (clipped into the table)
    hi = np.searchsorted(_POS, np.minimum(a, E4M3_MAX), side="left")
    hi = np.clip(hi, 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo = a - _POS[lo]
    d_hi = _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((hi & 1) == 0))
    mag = np.where(pick_hi, hi, lo)
    mag = np.where(a >= E4M3_MAX, 126, mag)
    code = (mag | np.where(neg, 0x80, 0)).astype(np.uint8)
    nan = np.isnan(y)
    if nan.any():
        code[nan] = np.uint8(0x7F)
    return code


# ---------------------------------------------------------------------------------------
# INT8 with scale and zero point ([KVPaged] "KV quantization: FP8 and INT8": one byte per
# element, needs a scale and a zero point). Affine code: value = (code - zero) * scale.
# ---------------------------------------------------------------------------------------
def int8_encode(y: np.ndarray, zero) -> np.ndarray:
    """float32 y = x / scale (already divided) -> int8 code = clip(round(y) + zero, -128, 127),
    round half to even."""
    y = np.asarray(y, dtype=np.float32)
    r = np.rint(y.astype(np.float64)) + np.asarray(zero, dtype=np.float64)
    return np.clip(r, -128, 127).astype(np.int8)


def int8_decode(codes: np.ndarray, zero) -> np.ndarray:
    """int8 codes -> (code - zero) as float64 (exact); multiply by the scale to dequantise."""
    return np.asarray(codes, dtype=np.int8).astype(np.float64) - np.asarray(zero, dtype=np.float64)
