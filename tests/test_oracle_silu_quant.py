"""Pins of the oracle's expert-side SiLU + block-fp8 quantiser.

"Lower latency and higher throughput with multi-node DeepSeek deployment",
section "Quantização": the activation kernel computes SiLU and quantises it
with one scale per 128-element block, working only on the rows the routing
counts populate.

The activation of a (gate, up) pair is defined as the binary32 number nearest
to the real value silu(g) * u = g u / (1 + e^-g), ties to even.  It is pinned
against 50-digit decimal arithmetic (Python's decimal module, whose exp is
correctly rounded) on every finite bf16 gate value and on sampled pairs, and
against an fp64 evaluation on every gate value times many up values; the
quantiser and the row selection are pinned by properties.
"""
import math
from decimal import Context, Decimal

import numpy as np
import pytest

import oracle
from tests._lib import silu_pairs_near_rounding_boundaries
from workloads import bf16_bits_to_f32, f32_to_bf16_bits

DEC = Context(prec=50, Emax=10**6, Emin=-10**6)


def _finite_bf16_bits():
    bits = np.arange(0, 0x10000, dtype=np.uint32)
    return bits[((bits >> 7) & 0xFF) != 0xFF].astype(np.uint16)


def _nearest_f32(D: Decimal) -> np.float32:
    """The binary32 number nearest to the decimal D (ties to even).

    float(D) rounds D to binary64 correctly, and binary64 rounding keeps order,
    so rounding that double to binary32 gives the nearest binary32 of D unless
    the double is itself halfway between two binary32 numbers; then the exact
    comparison of D with that halfway point decides.
    """
    m = float(D)
    f = np.float32(m)
    if float(f) != m:
        n = np.nextafter(f, np.float32(math.copysign(np.inf, m - float(f))))
        if (float(f) + float(n)) / 2 == m:           # m is a binary32 halfway point
            d = D - Decimal(m)
            assert d != 0                            # the real value is never halfway
            toward_n = (d > 0) == (float(n) > float(f))
            f = n if toward_n else f
    return f


def _exact_activation(g: float, u: float) -> np.float32:
    """RN_binary32(g u / (1 + e^-g)) from 50-digit decimal arithmetic.

    Outside |g| <= 200 the tails are closed forms: for g > 200 the quotient
    differs from g u by a relative e^-200, and g u (a product of two 8-bit
    significands) is a binary32 number, so it is the result; for g < -200,
    |silu(g) u| < 200 e^-200 * 3.4e38 < 2^-150, so the result is a zero with the
    sign of g u.
    """
    sign_zero = np.float32(math.copysign(0.0, g) * math.copysign(1.0, u))
    if g == 0 or u == 0:
        return sign_zero
    if g > 200:
        with np.errstate(over="ignore"):
            return np.float32(g * u)
    if g < -200:
        return sign_zero
    G, U = Decimal(g), Decimal(u)
    D = DEC.divide(DEC.multiply(G, U), DEC.add(1, DEC.exp(-G)))
    return _nearest_f32(D)


def _same(a, b) -> bool:
    return np.float32(a).view(np.uint32) == np.float32(b).view(np.uint32)


def test_activation_is_correctly_rounded_on_every_bf16_gate():
    bits = _finite_bf16_bits()
    g = bf16_bits_to_f32(bits)
    for ubits in (0x3F80, 0xC0A3):                  # u = 1 and u = -5.09375
        got = oracle.silu_mul_bits(bits, np.full(bits.shape, ubits, np.uint16))
        u = float(bf16_bits_to_f32(np.uint16(ubits)))
        bad = [float(gi) for gi, a in zip(g, got) if not _same(a, _exact_activation(float(gi), u))]
        assert not bad, bad[:10]


def test_activation_is_correctly_rounded_on_sampled_pairs():
    # pairs over the whole exponent range, including results that are binary32
    # subnormals, results near the binary32 limit, and bf16 subnormal inputs
    rng = np.random.default_rng(11)
    n = 6000
    gb = f32_to_bf16_bits((rng.standard_normal(n) * np.exp2(rng.integers(-10, 8, n))).astype(np.float32))
    ue = rng.integers(-133, 100, n).astype(np.float64)
    ub = f32_to_bf16_bits((rng.uniform(1, 2, n) * np.exp2(ue) * rng.choice([-1, 1], n)).astype(np.float32))
    gb[:200] = f32_to_bf16_bits(rng.uniform(-180, -60, 200).astype(np.float32))   # tiny results
    got = oracle.silu_mul_bits(gb, ub)
    g, u = bf16_bits_to_f32(gb), bf16_bits_to_f32(ub)
    assert np.any((got != 0) & (np.abs(got) < 2.0 ** -126))      # subnormal results occur
    for i in range(n):
        want = _exact_activation(float(g[i]), float(u[i]))
        assert _same(got[i], want), (float(g[i]), float(u[i]), float(got[i]), float(want))


def test_activation_is_correctly_rounded_next_to_rounding_boundaries():
    # pairs whose value lies within 2^-36 of a binary32 halfway point, many of
    # them closer than an fp64 evaluation resolves (small gates, where
    # silu(g) = g/2 + g^2/4 - ...); the up value is also scaled by powers of two
    gb, ub = silu_pairs_near_rounding_boundaries()
    assert len(gb) > 500
    for shift in (0, 40, -60):
        us = ub.astype(np.int32) + (shift << 7)       # u * 2^shift (exponent field)
        got = oracle.silu_mul_bits(gb, us.astype(np.uint16))
        g, u = bf16_bits_to_f32(gb), bf16_bits_to_f32(us.astype(np.uint16))
        for i in range(len(gb)):
            assert _same(got[i], _exact_activation(float(g[i]), float(u[i]))), (float(g[i]), float(u[i]))


def test_activation_within_half_ulp_of_fp64_on_every_gate_and_many_up_values():
    bits = _finite_bf16_bits()
    g64 = bf16_bits_to_f32(bits).astype(np.float64)
    keep = np.abs(g64) <= 700
    bits, g64 = bits[keep], g64[keep]
    rng = np.random.default_rng(5)
    for ub in f32_to_bf16_bits(rng.standard_normal(32).astype(np.float32) * 3):
        u = float(bf16_bits_to_f32(np.uint16(ub)))
        got = oracle.silu_mul_bits(bits, np.full(bits.shape, ub, np.uint16)).astype(np.float64)
        with np.errstate(over="ignore"):
            a64 = g64 * u / (1.0 + np.exp(-g64))
        half_ulp = np.maximum(np.spacing(np.abs(a64).astype(np.float32)).astype(np.float64), 2.0 ** -149) / 2
        assert np.all(np.abs(got - a64) <= half_ulp + np.abs(a64) * 2.0 ** -50), u


def test_activation_signs_zeros_and_tails():
    for g, u in [(0.0, 3.0), (-0.0, 3.0), (0.0, -3.0), (-0.0, -3.0), (2.0, 0.0), (-2.0, 0.0),
                 (2.0, -0.0), (-2.0, -0.0)]:
        assert _same(oracle.silu_mul(g, u), np.float32(math.copysign(0.0, g) * math.copysign(1.0, u)))
    for g in [100.0, 201.0, 1000.0, 3.0e38]:
        assert oracle.silu_mul(g, 1.0) == np.float32(g)             # 1 + e^-g is 1 to 2^-144
    assert _same(oracle.silu_mul(-200.5, 3.0e38), np.float32(-0.0))
    assert oracle.silu_mul(-150.0, 3.0e38) < -1e-26                  # still a normal number
    rng = np.random.default_rng(1)
    for g in rng.uniform(-20, 20, 2000).astype(np.float32):
        # g sigmoid(g) - (-g) sigmoid(-g) = g
        d = oracle.silu_mul(float(g)) - oracle.silu_mul(float(-g))
        assert abs(d - float(g)) <= 2 * float(np.spacing(np.float32(max(abs(g), 1e-30))))


def _decode(c):
    c = np.asarray(c, np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    f, m = (c >> 3) & 0xF, c & 0x7
    return s * np.where(f == 0, m * 2.0 ** -9, (1 + m / 8.0) * np.exp2(f - 7.0))


def _problem(rows, I, seed):
    rng = np.random.default_rng(seed)
    gu = f32_to_bf16_bits((rng.standard_normal((rows, 2 * I)) * 2).astype(np.float32))
    src = np.arange(rows, dtype=np.int32)
    src[rng.random(rows) < 0.2] = -1            # padding rows
    return gu, src


def test_rows_selected_by_routing_and_in_use_count():
    gu, src = _problem(50, 256, 2)
    act, scale = oracle.silu_quant(gu, src, rows_in_use=40, fill=0xA5)
    for r in range(50):
        written = r < 40 and src[r] >= 0
        assert np.all(act[r] == 0xA5) != written, r


def test_quantised_activation_properties():
    gu, src = _problem(20, 512, 3)
    src[:] = np.arange(20)
    act, scale = oracle.silu_quant(gu, src, rows_in_use=20)
    a32 = oracle.silu_mul_bits(gu[:, :512], gu[:, 512:])
    g = bf16_bits_to_f32(gu[:, :512]).astype(np.float64)
    u = bf16_bits_to_f32(gu[:, 512:]).astype(np.float64)
    a64 = g * u / (1.0 + np.exp(-g))
    assert np.all(np.abs(a32 - a64) <= 2.0 ** -24 * np.abs(a64) + 1e-40)
    for r in range(20):
        for b in range(4):
            blk = a32[r, 128 * b:128 * (b + 1)].astype(np.float64)
            amax = np.abs(blk).max()
            assert abs(scale[r, b] * 448.0 - amax) <= amax * 2.0 ** -23
            i = int(np.abs(blk).argmax())
            assert act[r, 128 * b + i] == (0xFE if blk[i] < 0 else 0x7E)
            deq = _decode(act[r, 128 * b:128 * (b + 1)]) * float(scale[r, b])
            q = np.abs(blk) / float(scale[r, b])
            half = np.where(q < 2.0 ** -6, 2.0 ** -10,
                            np.exp2(np.floor(np.log2(np.maximum(q, 2.0 ** -6))) - 4)) * float(scale[r, b])
            assert np.all(np.abs(deq - blk) <= half * (1 + 1e-6) + np.abs(blk) * 2.0 ** -23)


@pytest.mark.parametrize("in_use", [33, 20])
def test_column_major_scales_are_the_transpose(in_use):
    # the column-major stride is the row capacity, whatever the rows in use
    gu, src = _problem(33, 384, 4)
    a1, s1 = oracle.silu_quant(gu, src, rows_in_use=in_use, fill=0)
    a2, s2 = oracle.silu_quant(gu, src, rows_in_use=in_use, col_major=True, fill=0)
    np.testing.assert_array_equal(a1, a2)
    np.testing.assert_array_equal(s1.T, s2)
