"""Parity at the full workload sizes, in the launch configuration bench.py
times (eps 1e-5, LayerNorm without affine parameters), on sampled outputs the
oracle computes one by one:

- every row's LayerNorm statistics and the tensor scale (the oracle runs the
  LayerNorm over the whole tensor for the tensor scale anyway);
- mask indices, codes and scales of sampled rows, bit for bit (the oracle
  prepares the sampled rows with the whole tensor's scale);
- weight codes and both scale views of sampled weight rows, bit for bit;
- GEMM outputs at sampled (row, column) pairs within 1e-3 * sum|a||w|.

Workloads: the Llama-3.1-8B layer set at M = 8192 (the benchmark step), the
Qwen2.5-7B shapes at M = 4096 for NVFP4/MXFP4 x 2:4/4:8, and the
down-projection sweep over M and outlier fractions.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import assert_bits_equal, assert_linear_close, cuda16

pytestmark = pytest.mark.gpu

EPS = 1e-5


@pytest.fixture(scope="module")
def sq():
    import sparsity_gemm_b200 as sq
    assert torch.cuda.is_available()
    sq.lib()
    return sq


def _sample(n, count, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.r_[0, n - 1, rng.choice(n, size=min(count, n), replace=False)])


def _oracle_stats_and_scale(x, fmt):
    """Per-row (mu, rstd) of every row and the tensor scale, by the oracle's
    LayerNorm over the whole tensor in row chunks."""
    rows, k = x.shape
    mu = np.empty(rows, np.float32)
    rstd = np.empty(rows, np.float32)
    amax = np.float32(0)
    step = max(1, (1 << 24) // k)
    for r0 in range(0, rows, step):
        m_, r_ = oracle.ln_stats(x[r0:r0 + step], EPS)
        mu[r0:r0 + step], rstd[r0:r0 + step] = m_, r_
        xl = oracle.ln_apply(x[r0:r0 + step], None, None, m_, r_)
        amax = max(amax, np.abs(xl).max())
    return mu, rstd, oracle.tensor_scale(np.array([amax], np.float32), fmt)


def check_prep(sq, x, fmt, n, m, rows):
    p = sq.prepare(cuda16(x), None, None, EPS, n, m, fmt)
    ex = sq.prep_export(p)
    mu, rstd, s_t = _oracle_stats_and_scale(x, fmt)
    assert_bits_equal("mu (all rows)", ex["mu"], mu)
    assert_bits_equal("rstd (all rows)", ex["rstd"], rstd)
    assert_bits_equal("s_t", np.float32([ex["s_t"]]), np.float32([s_t]))
    op = oracle.prepare(x[rows], None, None, EPS, n, m, fmt, s_t=s_t)
    for name, key, want in [("mask idx", "idx", op.idx), ("S codes", "s_codes", op.s_codes),
                            ("S scales", "s_scales", op.s_scales), ("R codes", "r_codes", op.r_codes),
                            ("R scales", "r_scales", op.r_scales)]:
        assert_bits_equal(name, ex[key][rows], want)
    return p, op


def check_weight(sq, w, fmt, rows):
    qw = sq.quantize_weight(cuda16(w), fmt)
    wx = sq.weight_export(qw)
    amax = np.float32(np.abs(w.astype(np.float32)).max())
    s_tw = oracle.tensor_scale(np.array([amax], np.float32), fmt)
    assert_bits_equal("s_tW", np.float32([wx["s_tw"]]), np.float32([s_tw]))
    codes, scales = oracle.quantize(w[rows].astype(np.float32), fmt, s_tw)
    assert_bits_equal("W codes", wx["codes"][rows], codes)
    assert_bits_equal("W scales (backbone view)", wx["scales"][rows], scales)
    assert_bits_equal("W scales (residual view)", wx["scales_residual"][rows], scales)
    return qw, codes, scales, s_tw


def check_linear(sq, p, op, a_sel, qw, w_codes, w_scales, s_tw, fmt, w_rows):
    """GPU output at rows rows[a_sel] (op holds the oracle's prepared rows)
    and columns w_rows, against the oracle."""
    out = sq.linear(p, qw).cpu().numpy()
    got = out[np.ix_(a_sel[1], w_rows)]
    want, bound = oracle.linear(op.s_codes[a_sel[0]], op.s_scales[a_sel[0]], op.r_codes[a_sel[0]],
                                op.r_scales[a_sel[0]], op.s_t, w_codes, w_scales, s_tw, fmt)
    assert_linear_close(got, want, bound)
    assert sq.get_last_error() == sq.OK


def run_layer_set(sq, ls, m_tok, fmt, n, m, preps_to_check=None, linears_to_check=None, seed=0):
    rows = _sample(m_tok, 12, seed)
    a_pick = np.arange(0, len(rows), max(1, len(rows) // 3))  # a few of the sampled rows for the GEMM
    a_sel = (a_pick, rows[a_pick])
    prepared = {}
    for i, (name, k) in enumerate(ls.preps):
        if preps_to_check is not None and name not in preps_to_check:
            continue
        x = synth.activations_student(i, m_tok, k)
        prepared[name] = check_prep(sq, x, fmt, n, m, rows)
    for j, lin in enumerate(ls.linears):
        if linears_to_check is not None and lin.name not in linears_to_check:
            continue
        w = synth.weights(1000 + j, lin.n_out, lin.k)
        w_rows = _sample(lin.n_out, 256, seed + j)
        qw, wc, wsc, s_tw = check_weight(sq, w, fmt, w_rows)
        p, op = prepared[lin.prep]
        check_linear(sq, p, op, a_sel, qw, wc, wsc, s_tw, fmt, w_rows)


def test_llama31_8b_layer_set_m8192_nvfp4_2of4(sq):
    """The benchmark step: 4 preparations and 7 linears at M = 8192."""
    run_layer_set(sq, synth.LLAMA31_8B, 8192, 0, 2, 4)


@pytest.mark.parametrize("fmt,n,m", [(0, 2, 4), (1, 2, 4), (0, 4, 8), (1, 4, 8)])
def test_qwen25_7b_m4096(sq, fmt, n, m):
    run_layer_set(sq, synth.QWEN25_7B, 4096, fmt, n, m, preps_to_check={"attn_in", "down_in"},
                  linears_to_check={"k_proj", "down_proj"}, seed=fmt * 10 + n)


def test_down_projection_sweep(sq):
    """Down projection 14336 -> 4096 over M (powers of two, 1 .. 16384) and
    outlier fractions 0.1%, 1%, 5% (a subset of the grid)."""
    k, n_out = 14336, 4096
    w = synth.weights(1006, n_out, k)
    w_rows = _sample(n_out, 128, 5)
    qw, wc, wsc, s_tw = check_weight(sq, w, 0, w_rows)
    for m_tok, frac in [(1, 0.01), (16, 0.001), (128, 0.05), (2048, 0.01), (16384, 0.05)]:
        x = synth.activations_student(6, m_tok, k, outlier_frac=frac)
        rows = _sample(m_tok, 6, m_tok)
        p, op = check_prep(sq, x, 0, 2, 4, rows)
        a_pick = np.arange(min(2, len(rows)))
        check_linear(sq, p, op, (a_pick, rows[a_pick]), qw, wc, wsc, s_tw, 0, w_rows)
