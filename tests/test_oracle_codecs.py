"""Pins of the oracle's storage codecs against the format definitions and library routines.

bf16: torch's CPU float32 -> bfloat16 conversion (round to nearest even) and hand-derived
ties. E4M3: the OCP definition's landmark values, torch's float8_e4m3fn (decode of every
code; encode of in-range values) and a brute-force nearest-value search.
"""
import numpy as np
import pytest
import torch

from oracle import codecs


def test_bf16_landmarks():
    x = np.array([1.0, -2.0, 0.0, -0.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20,
                  3.0e38, np.inf], dtype=np.float32)
    got = codecs.bf16_encode(x)
    # 1+2^-8 ties to even (down), 1+3*2^-8 ties to even (up), just above a tie rounds up,
    # 3e38 rounds to the largest finite bf16 neighbour or inf as RNE dictates.
    assert list(got[:7]) == [0x3F80, 0xC000, 0x0000, 0x8000, 0x3F80, 0x3F82, 0x3F81]
    assert got[8] == 0x7F80
    assert np.isnan(codecs.bf16_decode(codecs.bf16_encode(np.array([np.nan], np.float32))))[0]


def test_bf16_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200_000).astype(np.float32),
                        (rng.standard_normal(50_000) * 1e30).astype(np.float32),
                        (rng.standard_normal(50_000) * 1e-38).astype(np.float32)])
    # exact ties: bf16 value + half an ulp
    b = rng.integers(0, 0x7F00, 20_000).astype(np.uint32)
    ties = ((b << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(codecs.bf16_encode(x), ref)
    back = codecs.bf16_decode(ref)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16)
                          .to(torch.float64).numpy())


def test_e4m3_landmarks():
    t = codecs.E4M3_TABLE
    assert t[0x38] == 1.0
    assert t[0x7E] == 448.0                    # largest finite: 1.75 * 2^8
    assert t[0x01] == 2.0 ** -9                # smallest subnormal: 1/8 * 2^-6
    assert t[0x07] == 7 / 8 * 2.0 ** -6        # largest subnormal
    assert t[0x08] == 2.0 ** -6                # smallest normal
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.signbit(t[0x80]) and t[0x80] == 0.0
    fin = t[np.isfinite(t)]
    assert fin.size == 254
    assert np.all(np.diff(t[:127]) > 0)
    assert np.array_equal(t[0x80:0xFF], -t[0x00:0x7F])


def test_e4m3_decode_matches_torch_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = codecs.e4m3_decode(codes)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[fin], ref[fin])


def _brute_nearest(y):
    vals = codecs.E4M3_TABLE
    codes = [c for c in range(256) if np.isfinite(vals[c])]
    out = []
    for yy in y.astype(np.float64):
        if abs(yy) >= 448.0:
            out.append(0x7E | (0x80 if yy < 0 else 0))
            continue
        best, bd = None, None
        for c in codes:
            if (c & 0x80) != (0x80 if np.signbit(yy) else 0):
                continue
            dd = abs(yy - vals[c])
            if bd is None or dd < bd or (dd == bd and (c & 1) == 0):
                best, bd = c, dd
        out.append(best)
    return np.array(out, dtype=np.uint8)


def test_e4m3_encode_brute_force_and_ties():
    rng = np.random.default_rng(1)
    y = np.concatenate([rng.standard_normal(600) * 100, rng.standard_normal(300) * 0.01,
                        [0.0, -0.0, 2.0 ** -10, -(2.0 ** -10), 3 * 2.0 ** -10, 1.0625, 1.1875,
                         448.0, 455.0, 470.0, 1e6, -1e6, 2.0 ** -12]]).astype(np.float32)
    got = codecs.e4m3_encode(y)
    assert np.array_equal(got, _brute_nearest(y))
    # ties to even: 2^-10 is halfway between 0 and 2^-9 -> 0; 3*2^-10 halfway between
    # 2^-9 (code 1) and 2^-8 (code 2) -> code 2; 1.0625 between 1.0 (0x38) and 1.125 (0x39)
    # -> 0x38; 1.1875 between 1.125 and 1.25 (0x3A) -> 0x3A.
    assert list(got[-13:-6]) == [0x00, 0x80, 0x00, 0x80, 0x02, 0x38, 0x3A]
    assert list(got[-6:-1]) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]   # satfinite


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(2)
    y = np.concatenate([rng.standard_normal(300_000) * 60,
                        rng.uniform(-464, 464, 100_000),
                        rng.standard_normal(100_000) * 1e-3]).astype(np.float32)
    y = y[np.abs(y) < 464.0]
    # every midpoint between adjacent finite magnitudes (exact in float32)
    mags = codecs.E4M3_TABLE[:127]
    mids = ((mags[1:] + mags[:-1]) / 2).astype(np.float32)
    y = np.concatenate([y, mids, -mids])
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codecs.e4m3_encode(y), ref)


def test_e4m3_nan_encodes_to_a_nan_pattern():
    """The format has no infinities and its only NaN patterns are S.1111.111: NaN must encode
    to one of them (torch agrees on the positive one), never to a finite code."""
    y = np.array([np.nan], np.float32)
    c = codecs.e4m3_encode(y)
    assert np.isnan(codecs.e4m3_decode(c))[0] and (int(c[0]) & 0x7F) == 0x7F
    assert int(c[0]) == int(torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8)[0])


def test_e4m3_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = codecs.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(codecs.e4m3_encode(vals), codes)


def _brute_int8(y, zero):
    """Nearest code c in [-128, 127] to y + zero with ties to an even (c - zero), then clip."""
    out = []
    for yy, z in zip(np.asarray(y, np.float64).ravel(), np.broadcast_to(zero, np.shape(y)).ravel()):
        lo = int(np.floor(yy))
        cands = [lo, lo + 1]
        best = min(cands, key=lambda c: (abs(yy - c), c % 2))
        out.append(min(127, max(-128, best + int(z))))
    return np.array(out, dtype=np.int8).reshape(np.shape(y))


def test_int8_encode_brute_force_ties_and_clipping():
    rng = np.random.default_rng(3)
    y = np.concatenate([rng.uniform(-140, 140, 3000), np.arange(-130, 130) + 0.5,
                        [0.0, -0.0, 0.5, -0.5, 1.5, -1.5, 2.5, 1e9, -1e9]]).astype(np.float32)
    zero = rng.integers(-20, 21, y.shape).astype(np.int32)
    got = codecs.int8_encode(y, zero)
    assert np.array_equal(got, _brute_int8(y, zero))
    # ties go to the even integer before the zero point is added
    assert list(codecs.int8_encode(np.array([0.5, 1.5, 2.5, -0.5, -1.5], np.float32), 3)) == \
        [3, 5, 5, 3, 1]
    assert list(codecs.int8_encode(np.array([1e9, -1e9], np.float32), 0)) == [127, -128]


def test_int8_roundtrip_and_affine_decode():
    codes = np.arange(-128, 128).astype(np.int8)
    for zero in (-128, -7, 0, 9, 127):
        vals = codecs.int8_decode(codes, zero)            # code - zero, exact
        assert np.array_equal(vals, np.arange(-128, 128) - zero)
        assert np.array_equal(codecs.int8_encode(vals.astype(np.float32), zero), codes)
    # a block quantised with the min/max recipe maps its min and max to the range ends and
    # every value to within half a step of itself
    import workloads
    rng = np.random.default_rng(4)
    for _ in range(50):
        x = (rng.standard_normal((16, 128)) * rng.uniform(0.01, 50)).astype(np.float32)
        scale, zero = workloads._int8_params(x)
        c = codecs.int8_encode((x / scale).astype(np.float32), zero)
        back = codecs.int8_decode(c, zero) * float(scale)
        assert np.abs(back - x).max() <= 0.5 * float(scale) * (1 + 1e-5) + 1e-7
        assert c.min() <= -127 and c.max() >= 126
