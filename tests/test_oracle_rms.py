"""Pins for the oracle's RMSNorm preparation (normalization by the root
mean square, no centring, the form the evaluated model families use):

- rows that sum to exactly zero have mu = 0 under LayerNorm too, so with a
  power-of-two K the RMSNorm statistics and every prepared output equal the
  LayerNorm ones bit for bit (the LayerNorm statistics are pinned against
  exact rationals elsewhere);
- scaling a row by 2 (with eps negligible against the mean square) leaves
  every prepared output unchanged, which a wrong power of the mean square,
  a missing or extra factor of K, or any centring would break;
- the normalized values agree with torch's rms_norm in binary64 within the
  two binary32 roundings of rstd and of the product;
- the mean square equals the variance plus the squared mean: 1/rstd^2 of
  the two forms differ by mu^2 (so rstd_rms <= rstd_ln).
"""
import numpy as np
import pytest
import torch

import synth

KEYS = ["mu", "rstd", "x_ln", "idx", "s_codes", "s_scales", "r_codes", "r_scales"]


def _zero_sum_rows(seed, rows, k):
    """Rows of k fp16 values: k/2 random values and their negations, in a
    random order, so that every row sums to exactly zero."""
    rng = np.random.default_rng(seed)
    half = synth.activations_student(seed, rows, k // 2).view(np.float16)
    x = np.concatenate([half, -half], axis=1)
    for r in range(rows):
        x[r] = x[r, rng.permutation(k)]
    return x


@pytest.mark.parametrize("k,fmt,n,m", [(256, 0, 2, 4), (1024, 1, 4, 8)])
def test_zero_mean_rows_reduce_to_layernorm(orc, k, fmt, n, m):
    x = _zero_sum_rows(90 + k, 6, k)
    assert np.all(x.view(np.float16).astype(np.float64).sum(axis=1) == 0)
    g = synth.ln_params(91, k)[0]
    for gamma in (None, g):
        a = orc.prepare(x, gamma, None, 1e-5, n, m, fmt, norm="rms")
        b = orc.prepare(x, gamma, None, 1e-5, n, m, fmt, norm="layer")
        for key in KEYS:
            assert np.array_equal(np.asarray(getattr(a, key)).view(np.uint8),
                                  np.asarray(getattr(b, key)).view(np.uint8)), key
        assert a.s_t == b.s_t


@pytest.mark.parametrize("fmt", [0, 1])
def test_power_of_two_scaling_leaves_outputs_unchanged(orc, fmt):
    k = 512
    x = synth.activations_student(92, 5, k)
    xf = x.view(np.float16).astype(np.float32)
    assert np.abs(xf).max() * 2 < 65504
    x2 = (xf * 2).astype(np.float16)
    eps = 1e-30  # negligible against the mean square in binary64
    a = orc.prepare(x, None, None, eps, 2, 4, fmt, norm="rms")
    b = orc.prepare(x2, None, None, eps, 2, 4, fmt, norm="rms")
    assert np.array_equal(b.rstd, a.rstd / 2)
    for key in ["x_ln", "idx", "s_codes", "s_scales", "r_codes", "r_scales"]:
        assert np.array_equal(np.asarray(getattr(a, key)), np.asarray(getattr(b, key))), key
    assert a.s_t == b.s_t


def test_agrees_with_torch_rms_norm(orc):
    k = 2048
    x = synth.activations_student(93, 8, k)
    g = synth.ln_params(94, k)[0]
    p = orc.prepare(x, g, None, 1e-5, 2, 4, 0, norm="rms")
    xt = torch.from_numpy(x.view(np.float16).astype(np.float64))
    gt = torch.from_numpy(g.view(np.float16).astype(np.float64))
    ref = torch.nn.functional.rms_norm(xt, (k,), weight=gt, eps=1e-5).numpy()
    err = np.abs(p.x_ln.astype(np.float64) - ref)
    # rstd and each of the two products round once to binary32 (2^-24 each)
    assert np.all(err <= 2.0 ** -22 * np.abs(ref) + 1e-30), err.max()


def test_mean_square_is_variance_plus_squared_mean(orc):
    """1/rstd_rms^2 - eps = 1/rstd_ln^2 - eps + mu^2 (mean square = variance
    + squared mean), to the binary32 rounding of the two rstd values; hence
    rstd_rms <= rstd_ln, strictly once the mean matters."""
    k = 768
    x = synth.activations_student(95, 16, k)
    shifted = (x.view(np.float16).astype(np.float32) + 64.0).astype(np.float16)
    eps = 1e-5
    for rows in (x, shifted):
        _, r_rms = orc.rms_stats(rows, eps)
        mu, r_ln = orc.ln_stats(rows, eps)
        ms = 1.0 / r_rms.astype(np.float64) ** 2 - eps
        want = 1.0 / r_ln.astype(np.float64) ** 2 - eps + mu.astype(np.float64) ** 2
        assert np.all(np.abs(ms - want) <= 4 * 2.0 ** -23 * ms), np.abs(ms - want).max()
        assert np.all(r_rms <= r_ln)
    mu, _ = orc.ln_stats(shifted, eps)
    assert np.all(orc.rms_stats(shifted, eps)[1] < orc.ln_stats(shifted, eps)[1])
