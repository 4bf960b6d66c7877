"""The certified statistics of the warp-per-row kernel (rows longer than 2048
elements), checked on the CPU against the oracle.

The kernel sums x^2 in binary64 in its own order (lane l takes the 8-element
vectors l, l + 32, ...; within a vector the even elements go to one
accumulator and the odd ones to another; the two are joined and then summed
over the 32 lanes by a butterfly), bounds the error of that sum by
(K/32 + 8) 2^-51 times the computed value, and accepts rstd only where both
ends of the bound give the same binary32 value. These tests replay that
order with numpy binary64 arithmetic (each square is exact, each addition
rounds once, as the kernel's FMA does) and check that the exact sum always
lies inside the bound, that every accepted row has the oracle's statistics
bit for bit, and that ordinary rows are accepted while degenerate ones are
left to the exact method.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import synth


def _kernel_order_sums(x: np.ndarray):
    """Per row: S1 = sum x 2^24 (exact integer) and the binary64 sum of x^2 in
    the kernel's order, for every lane after the butterfly (all equal)."""
    rows, k = x.shape
    xd = x.astype(np.float64).reshape(rows, k // 256, 32, 8)  # [row, j, lane, element]
    s2a = np.zeros((rows, 32))
    s2b = np.zeros((rows, 32))
    for j in range(k // 256):
        for p in range(4):
            s2a = s2a + xd[:, j, :, 2 * p] ** 2
            s2b = s2b + xd[:, j, :, 2 * p + 1] ** 2
    lanes = s2a + s2b
    for o in (16, 8, 4, 2, 1):
        lanes = lanes + lanes[:, np.arange(32) ^ o]
    assert np.all(lanes == lanes[:, :1])
    a = (x.astype(np.float64) * 2.0 ** 24).astype(np.int64)
    s1 = [int(v) for v in a.sum(axis=1)]
    s2_exact = [sum(int(v) * int(v) for v in row) for row in a]
    return s1, lanes[:, 0], s2_exact


def _finish(s1: int, d: int, k: int, eps: float, rms: bool):
    e = float(np.float32(eps))
    if rms:
        ms = float(d) / (k * 2.0 ** 48)
        return 0.0, float(np.float32(1.0 / math.sqrt(ms + e)))
    mean = float(s1) / (k * 2.0 ** 24)
    var = float(d) / (float(k * k) * 2.0 ** 48)
    return float(np.float32(mean)), float(np.float32(1.0 / math.sqrt(var + e)))


def _certify(s1: int, s2: float, k: int, eps: float, rms: bool):
    err = math.nextafter(s2 * (k // 32 + 8) * 2.0 ** -51, math.inf)
    lo = math.floor(Fraction(math.nextafter(s2 - err, -math.inf)) * 2 ** 48)
    hi = math.ceil(Fraction(math.nextafter(s2 + err, math.inf)) * 2 ** 48)
    lo = max(lo, 0)
    if rms:
        a, b = _finish(s1, lo, k, eps, True), _finish(s1, hi, k, eps, True)
    else:
        a = _finish(s1, max(k * lo - s1 * s1, 0), k, eps, False)
        b = _finish(s1, max(k * hi - s1 * s1, 0), k, eps, False)
    return lo, hi, a, a[1] == b[1]


def _rows(k: int) -> np.ndarray:
    x = synth.activations_student(940 + k, 20, k)
    x[0] = np.float16(3.5)                        # constant row: D = 0
    x[1, ::2] = np.float16(65504.0)               # extremes of both signs
    x[1, 1::2] = np.float16(-65504.0)
    x[2] = np.float16(1000.0)                     # large mean over a small spread
    x[2, ::7] = np.float16(1000.5)
    x[3] = 0
    x[4].view(np.uint16)[:] = np.arange(k, dtype=np.uint16) % 64 + 1  # fp16 subnormals
    x[5, : k // 2] = np.float16(65504.0)
    return x


@pytest.mark.parametrize("k", [4096, 14336])
@pytest.mark.parametrize("norm", ["layer", "rms"])
def test_certified_rows_match_the_oracle(orc, k, norm):
    import oracle
    x = _rows(k)
    rms = norm == "rms"
    mu, rstd = (oracle.rms_stats if rms else oracle.ln_stats)(x, 1e-5)
    s1, s2, s2_exact = _kernel_order_sums(x)
    accepted = []
    for r in range(x.shape[0]):
        lo, hi, st, ok = _certify(s1[r], float(s2[r]), k, 1e-5, rms)
        assert lo <= s2_exact[r] <= hi, r
        if ok:
            assert st[1] == float(rstd[r]) and (rms or st[0] == float(mu[r])), r
        accepted.append(ok)
    assert all(accepted[6:])                      # Student-t rows: decided by the bound
    if not rms:
        assert not accepted[0] and not accepted[2]  # left to the exact sums
