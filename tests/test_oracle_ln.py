"""Pins for the oracle's LayerNorm: exact rational statistics, a library
LayerNorm in fp64, closed-form special rows, and order independence."""
import decimal
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth


def _ulp32(v: float) -> float:
    v = np.float32(abs(v))
    return float(np.nextafter(v, np.float32(np.inf)) - v)


def _exact_stats(row16: np.ndarray, eps: np.float32):
    vals = [Fraction(float(v)) for v in row16.astype(np.float64)]
    k = len(vals)
    mean = sum(vals) / k
    var = sum((v - mean) ** 2 for v in vals) / k
    with decimal.localcontext() as ctx:
        ctx.prec = 60
        t = decimal.Decimal(var.numerator) / decimal.Decimal(var.denominator) + decimal.Decimal(float(eps))
        rstd = float(1 / t.sqrt())
    return mean, rstd


def _rows():
    rng = np.random.default_rng(0)
    yield synth.activations_gaussian(0, 4, 256, 4, 50.0)
    yield synth.activations_student(3, 3, 512)
    yield (rng.standard_normal((3, 64)) * 1e3).astype(np.float16)
    yield np.full((1, 64), np.float16(65504.0))
    tiny = np.zeros((1, 64), np.float16)
    tiny.view(np.uint16)[0, ::2] = np.arange(1, 33, dtype=np.uint16)  # fp16 subnormals
    yield tiny
    mix = np.zeros((1, 4096), np.float16)
    mix[0, 0::2] = 65504.0
    mix[0, 1::2] = -2.0 ** -24
    yield mix


@pytest.mark.parametrize("eps", [1e-5, 1e-6])
def test_stats_match_exact_rationals(orc, eps):
    eps32 = np.float32(eps)
    for x in _rows():
        mu, rstd = orc.ln_stats(x, eps)
        for r in range(x.shape[0]):
            mean, rs = _exact_stats(x[r], eps32)
            assert abs(float(mu[r]) - float(mean)) <= _ulp32(float(mean)) + 1e-45
            assert abs(float(rstd[r]) - rs) <= 1.5 * _ulp32(rs)


def _reading_stats(row16: np.ndarray, eps32: np.float32, norm: str):
    """The statistics' rounding sequence as the library documents it (exact
    integer sums of a = x 2^24; then each step one IEEE binary64 operation,
    as Python floats are, and one rounding to binary32):
      LayerNorm: mu = RN32(RN64(S1) / (K 2^24)),
                 rstd = RN32(1 / sqrt(RN64(K S2 - S1^2) / (K^2 2^48) + eps));
      RMSNorm:   rstd = RN32(1 / sqrt(RN64(S2) / (K 2^48) + eps)), mu = 0."""
    a = [int(Fraction(float(v)) * 2 ** 24) for v in row16.astype(np.float64)]
    k = len(a)
    s1 = sum(a)
    s2 = sum(v * v for v in a)
    if norm == "layer":
        mu = np.float32(float(s1) / float(k * 2 ** 24))
        var = float(k * s2 - s1 * s1) / float(k * k * 2 ** 48)
    else:
        mu = np.float32(0.0)
        var = float(s2) / float(k * 2 ** 48)
    return mu, np.float32(1.0 / math.sqrt(var + float(eps32)))


@pytest.mark.parametrize("norm", ["layer", "rms"])
@pytest.mark.parametrize("eps", [1e-5, 1e-6])
def test_stats_bit_exact_to_the_documented_rounding_sequence(orc, norm, eps):
    """Bit for bit: the oracle's statistics equal the documented sequence
    recomputed here with Python integers and IEEE binary64 operations (the
    rational pin above bounds that sequence against the exact values)."""
    eps32 = np.float32(eps)
    rows = list(_rows()) + [synth.activations_student(7, 5, 14336)]
    big = np.full((1, 16384), np.float16(65504.0))
    big[0, 1::3] = -65504.0
    rows.append(big)
    for x in rows:
        mu, rstd = (orc.ln_stats if norm == "layer" else orc.rms_stats)(x, eps)
        for r in range(x.shape[0]):
            want_mu, want_rstd = _reading_stats(x[r], eps32, norm)
            assert np.float32(mu[r]).view(np.uint32) == want_mu.view(np.uint32), (norm, r, mu[r], want_mu)
            assert np.float32(rstd[r]).view(np.uint32) == want_rstd.view(np.uint32), (norm, r, rstd[r], want_rstd)


def test_large_row_exercises_wide_sums(orc):
    # S2 near 2^94: K = 16384 entries of magnitude 65504 (a_i ~ 2^40)
    x = np.full((1, 16384), np.float16(65504.0))
    x[0, 1::3] = -65504.0
    mu, rstd = orc.ln_stats(x, 1e-5)
    mean, rs = _exact_stats(x[0], np.float32(1e-5))
    assert abs(float(mu[0]) - float(mean)) <= _ulp32(float(mean))
    assert abs(float(rstd[0]) - rs) <= 1.5 * _ulp32(rs)


def test_constant_and_alternating_rows(orc):
    c = np.full((1, 128), np.float16(3.5))
    mu, rstd = orc.ln_stats(c, 1e-5)
    assert mu[0] == np.float32(3.5)
    assert rstd[0] == np.float32(1.0 / np.sqrt(np.float64(np.float32(1e-5))))
    xl = orc.ln_apply(c, None, None, mu, rstd)
    assert np.all(xl == 0) and not np.any(np.signbit(xl))

    a = np.float16(1.5)
    alt = np.tile(np.array([a, -a], np.float16), 64)[None, :]
    mu, rstd = orc.ln_stats(alt, 1e-5)
    assert mu[0] == 0
    assert rstd[0] == np.float32(1.0 / np.sqrt(np.float64(2.25) + np.float64(np.float32(1e-5))))


def test_order_independent(orc):
    x = synth.activations_student(5, 2, 1024)
    mu, rstd = orc.ln_stats(x, 1e-5)
    perm = np.random.default_rng(1).permutation(1024)
    mu2, rstd2 = orc.ln_stats(x[:, perm], 1e-5)
    assert np.array_equal(mu, mu2) and np.array_equal(rstd, rstd2)


@pytest.mark.parametrize("affine", [False, True])
def test_apply_matches_library_layernorm(orc, affine):
    x = synth.activations_student(9, 8, 1024)
    g, b = synth.ln_params(9, 1024) if affine else (None, None)
    eps = 1e-5
    mu, rstd = orc.ln_stats(x, eps)
    got = orc.ln_apply(x, g, b, mu, rstd).astype(np.float64)
    xt = torch.from_numpy(x.astype(np.float64))
    w = None if g is None else torch.from_numpy(g.astype(np.float64))
    bb = None if b is None else torch.from_numpy(b.astype(np.float64))
    ref = torch.nn.functional.layer_norm(xt, (1024,), w, bb, eps=float(np.float32(eps))).numpy()
    gabs = np.ones(1024) if g is None else np.abs(g.astype(np.float64))
    babs = np.zeros(1024) if b is None else np.abs(b.astype(np.float64))
    # four binary32 roundings plus the rounding of mu and rstd
    tol = 2.0 ** -21 * ((np.abs(x.astype(np.float64)) + np.abs(mu[:, None])) * rstd[:, None] * gabs) \
        + 2.0 ** -22 * babs + 1e-30
    assert np.all(np.abs(got - ref) <= tol)


def test_apply_null_beta_keeps_negative_zero(orc):
    x = np.zeros((1, 16), np.float16)
    x.view(np.uint16)[0, 3] = 0x8000  # -0
    mu, rstd = orc.ln_stats(x, 1e-5)
    xl = orc.ln_apply(x, None, None, mu, rstd)
    assert np.signbit(xl[0, 3]) and not np.signbit(xl[0, 2])
