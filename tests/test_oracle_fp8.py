"""Pins of the oracle's e4m3 conversion and block quantiser.

The oracle converts a float to e4m3 by rounding onto the format's grid.  These
tests check it against things it does not compute itself: the OCP specification's
own table of points (tests/golden/e4m3_points.txt), a decoder written here from
the bit layout, exact midpoints between neighbouring codes, a brute-force nearest
search, and torch's float8_e4m3fn cast.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import f32_to_bf16_bits, bf16_bits_to_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_points.txt")


def decode(c: int) -> float:
    """Value of an e4m3 code from its bit fields (sign, 4-bit exponent, 3-bit mantissa)."""
    s = -1.0 if c & 0x80 else 1.0
    f, m = (c >> 3) & 0xF, c & 0x7
    if f == 0xF and m == 0x7:
        return math.nan
    if f == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (f - 7)


FINITE = [c for c in range(256) if not math.isnan(decode(c))]
POS = [c for c in range(0x7F)]  # 0x00 .. 0x7e: the non-negative finite codes, ascending


def test_golden_points_from_spec():
    rows = [ln.split() for ln in open(GOLDEN) if ln.strip() and not ln.startswith("#")]
    assert len(rows) >= 10
    for code_s, val_s in rows:
        code, val = int(code_s, 16), float(val_s)
        assert decode(code) == val and math.copysign(1, decode(code)) == math.copysign(1, val)
        assert oracle.e4m3_from_float(val) == code, (code_s, val_s)


def test_every_finite_code_round_trips():
    assert len(FINITE) == 254
    for c in FINITE:
        assert oracle.e4m3_from_float(decode(c)) == c, hex(c)


def test_positive_codes_are_ascending():
    vals = [decode(c) for c in POS]
    assert all(a < b for a, b in zip(vals, vals[1:]))


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_midpoints_round_to_even_code(sign):
    for c in POS[:-1]:
        lo, hi = decode(c), decode(c + 1)
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2  # exact in binary32
        even = c if c % 2 == 0 else c + 1
        sbit = 0x80 if sign < 0 else 0
        assert oracle.e4m3_from_float(sign * mid) == even | sbit
        below = np.nextafter(mid, np.float32(lo))
        above = np.nextafter(mid, np.float32(hi))
        assert oracle.e4m3_from_float(sign * below) == c | sbit
        assert oracle.e4m3_from_float(sign * above) == (c + 1) | sbit


def test_saturates_to_448():
    for v in [448.0, 448.5, 463.99, 464.0, 480.0, 1e4, 3.0e38]:
        assert oracle.e4m3_from_float(v) == 0x7E
        assert oracle.e4m3_from_float(-v) == 0xFE


def _brute_nearest(v: float) -> int:
    """Nearest finite code by exhaustive search; ties to the even code; clamp to 448."""
    a = min(abs(v), 448.0)
    best, bestd = None, None
    for c in POS:
        d = abs(decode(c) - a)
        if bestd is None or d < bestd or (d == bestd and c % 2 == 0):
            best, bestd = c, d
    if math.copysign(1.0, v) < 0:
        best |= 0x80
    return best


def test_brute_force_nearest_random():
    rng = np.random.default_rng(11)
    mags = np.exp2(rng.uniform(-14, 10, size=3000)).astype(np.float32)
    signs = rng.choice([-1.0, 1.0], size=mags.size).astype(np.float32)
    for v in (mags * signs):
        assert oracle.e4m3_from_float(float(v)) == _brute_nearest(float(v)), float(v)


def test_agrees_with_torch_cast_in_range():
    rng = np.random.default_rng(12)
    v = np.concatenate([
        rng.uniform(-448, 448, 20000),
        np.exp2(rng.uniform(-12, -5, 5000)) * rng.choice([-1, 1], 5000),
    ]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_from_float(float(a)) for a in v], dtype=np.uint8)
    np.testing.assert_array_equal(ours, ref)


# ---- block quantiser ---------------------------------------------------------

def _decode_codes(codes):
    return np.array([decode(int(c)) for c in codes])


def test_block_scale_and_amax_code():
    rng = np.random.default_rng(3)
    x = f32_to_bf16_bits(rng.standard_normal(7168).astype(np.float32))
    codes, scales = oracle.quantise_row_fp8(x)
    assert codes.shape == (7168,) and scales.shape == (56,)   # one scale per 128 values
    xf = bf16_bits_to_f32(x).reshape(56, 128)
    for b in range(56):
        amax = np.abs(xf[b]).max()
        # scale*448 recovers amax to within the rounding of one binary32 division
        assert abs(float(scales[b]) * 448.0 - amax) <= amax * 2.0 ** -23
        i = int(np.abs(xf[b]).argmax())
        assert codes[b * 128 + i] == (0xFE if xf[b, i] < 0 else 0x7E)


def test_dequantisation_error_bound():
    rng = np.random.default_rng(4)
    x = f32_to_bf16_bits((rng.standard_normal(1024) * np.exp2(rng.integers(-8, 8, 1024))).astype(np.float32))
    codes, scales = oracle.quantise_row_fp8(x)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    deq = _decode_codes(codes) * np.repeat(scales.astype(np.float64), 128)
    q = np.abs(xf) / np.repeat(scales.astype(np.float64), 128)
    # half the e4m3 grid spacing at q: 2^-10 below 2^-6, else 2^(floor(log2 q) - 4)
    half_ulp = np.where(q < 2.0 ** -6, 2.0 ** -10, np.exp2(np.floor(np.log2(np.maximum(q, 2.0 ** -6))) - 4))
    bound = half_ulp * np.repeat(scales.astype(np.float64), 128) * (1 + 1e-6) + np.abs(xf) * 2.0 ** -23
    assert np.all(np.abs(deq - xf) <= bound)


def test_zero_block_and_signed_zero():
    x = np.zeros(256, np.uint16)
    x[128:] = f32_to_bf16_bits(np.linspace(-1, 1, 128).astype(np.float32))
    x[0] = 0x8000  # -0.0 in an all-zero block still gives code +0
    x[130] = 0x8000  # -0.0 in a non-zero block keeps its sign
    codes, scales = oracle.quantise_row_fp8(x)
    assert scales[0] == 0.0 and np.all(codes[:128] == 0)
    assert scales[1] > 0 and codes[130] == 0x80


def test_blocks_are_independent():
    rng = np.random.default_rng(5)
    x = f32_to_bf16_bits(rng.standard_normal(512).astype(np.float32))
    c1, s1 = oracle.quantise_row_fp8(x)
    x2 = x.copy()
    x2[256:384] = f32_to_bf16_bits(rng.standard_normal(128).astype(np.float32) * 100)
    c2, s2 = oracle.quantise_row_fp8(x2)
    keep = np.r_[0:256, 384:512]
    np.testing.assert_array_equal(c1[keep], c2[keep])
    np.testing.assert_array_equal(s1[[0, 1, 3]], s2[[0, 1, 3]])


def test_tiny_and_subnormal_blocks():
    # bf16 subnormals: amax/448 is a binary32 subnormal; the division must still be exact-rounded
    x = np.array([1, 2, 3, 0x8001, 0x0080, 0x8005] + [0] * 122, np.uint16)
    codes, scales = oracle.quantise_row_fp8(x)
    xf = bf16_bits_to_f32(x)
    amax = np.float32(np.abs(xf).max())
    assert scales[0] == np.float32(amax) / np.float32(448.0) and scales[0] > 0
    for i in range(6):
        assert codes[i] == _brute_nearest(float(np.float32(xf[i]) / scales[0]))
