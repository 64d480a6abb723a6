"""The fast tier's SiLU gate table (combine_route_meta_b200/csrc/silu_table.inc).

The table holds, for each bf16 gate g with |g| in [2^-10, 2^3), the binary32
pair hi = RN(silu(g)), lo = RN(silu(g) - hi); the kernel's correctly rounded
activation rests on hi + lo lying within 2^-48 |silu(g)| of silu(g).  These
checks recompute silu(g) = g / (1 + e^-g) with 50-digit decimal arithmetic,
independently of the generator, and verify every entry against it.
"""
import math
import os
import re
import struct
import subprocess
import sys
from decimal import Context, Decimal

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "combine_route_meta_b200", "csrc")
DEC = Context(prec=50)


def _f(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", bits))[0]


def _pairs():
    text = open(os.path.join(CSRC, "silu_table.inc")).read()
    return [(int(a, 16), int(b, 16)) for a, b in re.findall(r"\{0x([0-9a-f]{8})u, 0x([0-9a-f]{8})u\}", text)]


def test_committed_table_is_what_the_generator_writes():
    r = subprocess.run([sys.executable, os.path.join(CSRC, "gen_silu_table.py"), "--check"])
    assert r.returncode == 0


def test_every_entry_is_the_rounded_pair_of_silu():
    pairs = _pairs()
    per_sign = 13 * 128 + 1
    assert len(pairs) == 2 * per_sign
    for sign in (0, 1):
        for e in range(13):
            for m in range(128):
                i = sign * per_sign + e * 128 + m
                gbits = (sign << 31) | ((e + 127 - 10) << 23) | (m << 16)
                g = Decimal(_f(gbits))
                s = DEC.divide(g, DEC.add(1, DEC.exp(-g)))
                hi, lo = _f(pairs[i][0]), _f(pairs[i][1])
                err = abs(DEC.subtract(DEC.add(Decimal(hi), Decimal(lo)), s))
                assert err <= abs(s) * Decimal(2) ** -48, (float(g), hi, lo)
                # hi is the nearest binary32 to silu(g): the rest is within half its ulp
                ulp = Decimal(2) ** (math.frexp(hi)[1] - 24)
                assert abs(DEC.subtract(s, Decimal(hi))) <= ulp / 2, float(g)
                assert abs(lo) <= float(ulp) / 2 * (1 + 2 ** -23)
        # the sentinel that gates outside the table index
        assert math.isnan(_f(pairs[sign * per_sign + 13 * 128][0]))


def test_table_sign_symmetry():
    # silu(-g) = silu(g) - g: the two signs' pairs agree with it to the table's precision
    pairs = _pairs()
    per_sign = 13 * 128 + 1
    for i in range(0, 13 * 128, 7):
        e, m = divmod(i, 128)
        g = _f(((e + 117) << 23) | (m << 16))
        pos = _f(pairs[i][0]) + _f(pairs[i][1])
        neg = _f(pairs[per_sign + i][0]) + _f(pairs[per_sign + i][1])
        assert abs((pos - g) - neg) <= 4 * 2 ** -48 * (abs(pos) + abs(g))
