"""The bracketed E2M1 encoding of the preparation kernels, checked on the CPU
with IEEE binary32 arithmetic (numpy rounds every float32 product and
quotient to nearest even and keeps subnormals).

The kernel encodes RN32(v / d) for a block step d in [2^-90, 2^90] without
dividing: with y = RN(1/d), ylo = RN(y (1 - 2^-21)) and yhi = RN(y (1 +
2^-21)), the products RN(v ylo) and RN(v yhi) lie strictly on either side
of v / d, so where their E2M1 codes agree that is the code of RN32(v / d);
elsewhere a correctly rounded quotient decides. These tests check the
bracketing and the agreement claim over the kernel's operand ranges, and
that the fallback stays rare on ordinary quotients. The E2M1 encoder is
ml_dtypes' (round to nearest even) after saturation to +-6.
"""
import ml_dtypes
import numpy as np

F32 = np.float32


def _e2m1(q: np.ndarray) -> np.ndarray:
    q = np.clip(q.astype(np.float32), F32(-6.0), F32(6.0))
    codes = q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    # the sign of zero results comes from the operand (the hardware
    # conversion keeps it); normalise the library's choice to that rule
    sign = (q.view(np.uint32) >> 31).astype(np.uint8)
    return (codes & 0x7) | (sign << 3)


def _divisors(rng, n):
    e = rng.integers(-90, 91, n)
    mant = rng.integers(0, 1 << 23, n, dtype=np.uint32)
    return ((e + 127).astype(np.uint32) << 23 | mant).view(np.float32)


def _bracket(v: np.ndarray, d: np.ndarray):
    with np.errstate(under="ignore", over="ignore"):
        y = F32(1.0) / d
        ylo = y * F32(1.0 - 2.0 ** -21)
        yhi = y * F32(1.0 + 2.0 ** -21)
        return v * ylo, v * yhi, v / d


def _quotient_cases(rng, n):
    d = _divisors(rng, n)
    kind = rng.integers(0, 4, n)
    q = np.empty(n, dtype=np.float64)
    # random quotients, log-uniform in [2^-12, 8]
    q[kind == 0] = 2.0 ** rng.uniform(-12, 3, (kind == 0).sum())
    # within 40 ulps of an E2M1 rounding boundary
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    t = ties[rng.integers(0, 7, (kind == 1).sum())]
    q[kind == 1] = (t.view(np.uint32) + rng.integers(-40, 41, t.size).astype(np.uint32)).view(np.float32)
    # exactly on a boundary (divisors with 19 significant bits, so that
    # the dividend t d is exact)
    q[kind == 2] = ties[rng.integers(0, 7, (kind == 2).sum())]
    d[kind == 2] = (d[kind == 2].view(np.uint32) & np.uint32(0xFFFFFFF0)).view(np.float32)
    # tiny quotients, down to the bottom of binary32
    q[kind == 3] = 2.0 ** rng.uniform(-160, -11, (kind == 3).sum())
    with np.errstate(under="ignore", over="ignore"):
        v = (q.astype(np.float32) * d).astype(np.float32)
    v = np.where(rng.integers(0, 2, n) == 1, -v, v)
    return v, d, kind


def test_products_bracket_the_quotient():
    rng = np.random.default_rng(20)
    v, d, _ = _quotient_cases(rng, 400_000)
    ql, qh, _ = _bracket(v, d)
    exact = v.astype(np.float64) / d.astype(np.float64)  # within 2^-53: far inside the 2^-22 margin
    normal = (np.abs(ql) >= F32(2.0 ** -126)) & (v != 0)
    pos, neg = normal & (v > 0), normal & (v < 0)
    assert pos.sum() > 100_000 and neg.sum() > 100_000
    assert np.all(ql[pos].astype(np.float64) < exact[pos]) and np.all(exact[pos] < qh[pos].astype(np.float64))
    assert np.all(ql[neg].astype(np.float64) > exact[neg]) and np.all(exact[neg] > qh[neg].astype(np.float64))


def test_agreeing_codes_are_the_code_of_the_rounded_quotient():
    rng = np.random.default_rng(21)
    v, d, kind = _quotient_cases(rng, 400_000)
    v[:64] = np.where(np.arange(64) % 2 == 0, F32(0.0), F32(-0.0))  # zero dividends of both signs
    ql, qh, q = _bracket(v, d)
    cl, ch, c = _e2m1(ql), _e2m1(qh), _e2m1(q)
    agree = cl == ch
    assert np.array_equal(cl[agree], c[agree])
    # zero dividends keep their sign through the products
    assert np.array_equal(cl[:64], np.where(np.arange(64) % 2 == 0, 0, 8).astype(np.uint8))
    # the fallback is taken near boundaries and on exact ties, rarely otherwise
    kind[:64] = -1
    assert np.array_equal(q[kind == 2].astype(np.float64), v[kind == 2].astype(np.float64) / d[kind == 2])
    assert (~agree[kind == 2]).all()
    assert (~agree[kind == 1]).any() and agree[kind == 1].any()
    assert (~agree[kind == 0]).mean() < 1e-3
    assert agree[kind == 3].all()
