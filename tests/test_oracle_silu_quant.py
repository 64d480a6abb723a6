"""Pins of the oracle's expert-side SiLU + block-fp8 quantiser.

"Lower latency and higher throughput with multi-node DeepSeek deployment",
section "Quantização": the activation kernel computes SiLU and quantises it
with one scale per 128-element block, working only on the rows the routing
counts populate.  The binary32 SiLU is pinned to double-precision mathematics
over every bf16 input; the quantiser and the row selection by properties.
"""
import math

import numpy as np
import pytest

import oracle
from workloads import bf16_bits_to_f32, f32_to_bf16_bits


def _silu64(g):
    return 0.0 if -g > 700 else g / (1.0 + math.exp(-g))


def _decode(c):
    c = np.asarray(c, np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    f, m = (c >> 3) & 0xF, c & 0x7
    return s * np.where(f == 0, m * 2.0 ** -9, (1 + m / 8.0) * np.exp2(f - 7.0))


def test_silu_matches_double_precision_on_every_bf16_value():
    bits = np.arange(0, 0x10000, dtype=np.uint32)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    for g in bf16_bits_to_f32(bits):
        s32, s64 = oracle.silu_f32(float(g)), _silu64(float(g))
        if abs(s64) > 1e-30:
            assert abs(s32 - s64) <= 2.0 * float(np.spacing(np.float32(abs(s64)))), float(g)
        else:
            assert abs(s32 - s64) <= 1e-36, float(g)


def test_silu_special_values_and_identity():
    assert oracle.silu_f32(0.0) == 0.0
    for g in [100.0, 1000.0, 3.0e38]:
        assert oracle.silu_f32(g) == np.float32(g)     # 1 + e^-g rounds to 1
    rng = np.random.default_rng(1)
    for g in rng.uniform(-20, 20, 2000).astype(np.float32):
        # g*sigmoid(g) - (-g)*sigmoid(-g) = g
        d = oracle.silu_f32(float(g)) - oracle.silu_f32(float(-g))
        assert abs(d - float(g)) <= 4 * float(np.spacing(np.float32(max(abs(g), 1e-30))))


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
    g = bf16_bits_to_f32(gu[:, :512]).astype(np.float64)
    u = bf16_bits_to_f32(gu[:, 512:]).astype(np.float64)
    a32 = np.array([[oracle.silu_f32(float(v)) for v in row] for row in bf16_bits_to_f32(gu[:, :512])],
                   np.float32) * bf16_bits_to_f32(gu[:, 512:])
    a64 = np.vectorize(_silu64)(g) * u
    assert np.all(np.abs(a32 - a64) <= 3e-7 * np.abs(a64) + 1e-30)
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
