"""Pins for the oracle's codecs against the format definitions and against an
independent library implementation (ml_dtypes), not against themselves."""
import math

import ml_dtypes
import numpy as np
import pytest

from conftest import read_golden


def test_half_decode_all_patterns(orc):
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    for b in range(0, 1 << 16, 7):  # every 7th pattern keeps the test fast
        v = orc.half_to_double(b)
        if math.isnan(ref[b]):
            assert math.isnan(v)
        else:
            assert v == ref[b] and math.copysign(1, v) == math.copysign(1, ref[b]), b


def test_e2m1_golden_table(orc):
    for y, code in read_golden("e2m1_rounding.txt"):
        assert orc.e2m1_encode(float(y)) == int(code), y


def test_e2m1_values_are_the_grid(orc):
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        v = orc.e2m1_value(c)
        assert abs(v) == grid[c & 7]
        assert math.copysign(1, v) == (-1 if c & 8 else 1)
        assert orc.e2m1_encode(v) == c  # round trip, -0 included


def _e2m1_library(y: np.ndarray) -> np.ndarray:
    return y.astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def test_e2m1_matches_library_on_ties_and_neighbours(orc):
    pts = []
    for t in [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 6.0, 0.0]:
        f = np.float32(t)
        for d in range(-3, 4):
            v = f
            step = np.float32(np.inf) if d > 0 else np.float32(-np.inf)
            for _ in range(abs(d)):
                v = np.nextafter(v, step)
            pts += [v, -v]
    pts = np.array(pts, np.float32)
    lib = _e2m1_library(pts)
    for y, c in zip(pts, lib):
        assert orc.e2m1_encode(float(y)) == int(c), float(y)


def test_e2m1_matches_library_random(orc):
    rng = np.random.default_rng(7)
    y = np.concatenate([rng.uniform(-8, 8, 20000), rng.standard_normal(5000) * 1e-3,
                        rng.uniform(-1e6, 1e6, 2000)]).astype(np.float32)
    lib = _e2m1_library(y)
    got = np.array([orc.e2m1_encode(float(v)) for v in y])
    assert np.array_equal(got, lib)


def test_ue4m3_golden_values(orc):
    for code, value in read_golden("ue4m3_values.txt"):
        assert orc.ue4m3_value(int(code)) == float(value)


def test_ue4m3_value_table_matches_library(orc):
    lib = np.arange(127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for c in range(127):
        assert orc.ue4m3_value(c) == lib[c]


def test_ue4m3_encode_matches_library(orc):
    rng = np.random.default_rng(11)
    # exact values, midpoints between neighbours, their float32 neighbours, random
    vals = [orc.ue4m3_value(c) for c in range(127)]
    mids = [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    pts = np.array(vals + mids + [2.0 ** -10, 2.0 ** -11, 1e-30, 0.0], np.float32)
    nb = np.concatenate([np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0))])
    rnd = np.exp(rng.uniform(np.log(1e-4), np.log(460), 20000)).astype(np.float32)
    u = np.concatenate([pts, nb, rnd])
    u = u[u <= 464.0]  # above 464 the library overflows to NaN; saturation is pinned below
    lib = u.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    got = np.array([orc.ue4m3_encode(float(v)) for v in u])
    assert np.array_equal(got, lib)


def test_ue4m3_saturates(orc):
    for u in [448.0, 464.0, 464.1, 480.0, 1e9, 3.0e38]:
        assert orc.ue4m3_encode(u) == 126


def test_mx_exponent_matches_frexp_and_library(orc):
    rng = np.random.default_rng(3)
    a = np.exp(rng.uniform(np.log(1e-38), np.log(3e38), 5000)).astype(np.float32)
    a = np.concatenate([a, np.float32([6.0, 7.999, 8.0, 1.0, 2.0 ** -126, 2.0 ** -149, 2.0 ** -140])])
    for v in a:
        m, ex = math.frexp(float(v))
        want = min(max(ex - 1 - 2, -127), 127)
        assert orc.mx_exponent(float(v)) == want
        # E8M0 holds 2^(e); the library's round trip of 2^e must give code e+127
        code = np.float32(2.0 ** want).astype(ml_dtypes.float8_e8m0fnu).view(np.uint8)
        assert int(code) == want + 127


def test_u128_to_double_correctly_rounded(orc):
    rng = np.random.default_rng(5)
    cases = [0, 1, 2 ** 53 - 1, 2 ** 53, 2 ** 53 + 1, 2 ** 53 + 2, 2 ** 53 + 3,
             2 ** 54 + 2, 2 ** 54 + 6, 2 ** 100 + 2 ** 47, 2 ** 100 + 2 ** 47 + 1,
             2 ** 100 + 3 * 2 ** 47, 2 ** 127 + 2 ** 74, (1 << 128) - 1 - (1 << 75)]
    for _ in range(2000):
        bits = int(rng.integers(1, 128))
        cases.append(int(rng.integers(0, 2 ** 62)) << max(0, bits - 62) | int(rng.integers(0, 2 ** 30)))
    for v in cases:
        v &= (1 << 128) - 1
        assert orc.u128_to_double(v) == float(v), v  # Python's int->float is correctly rounded
