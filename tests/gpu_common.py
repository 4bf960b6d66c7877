"""Helpers of the GPU parity tests: run the CUDA path (through the C ABI) and
the CPU oracle on the same seeded bytes and compare them."""
import numpy as np
import torch

import oracle
import sparsity_gemm_b200 as sq

FP16_FLOOR = 2.0 ** -24  # half an fp16 ulp at the subnormal end: output rounding floor


def cuda16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.float16)).cuda()


def first_diff(a, b):
    d = np.argwhere(a != b)
    return None if d.size == 0 else (tuple(d[0]), a[tuple(d[0])], b[tuple(d[0])], int(len(d)))


def assert_bits_equal(name, got, want):
    got = np.ascontiguousarray(got)
    want = np.ascontiguousarray(want)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    if got.dtype == np.float32:
        got, want = got.view(np.uint32), want.view(np.uint32)
    fd = first_diff(got, want)
    assert fd is None, f"{name}: first mismatch at {fd[0]}: gpu {fd[1]} oracle {fd[2]} ({fd[3]} mismatches)"


def gpu_prepare(x, gamma, beta, eps, n, m, fmt):
    g = None if gamma is None else cuda16(gamma)
    b = None if beta is None else cuda16(beta)
    p = sq.prepare(cuda16(x), g, b, eps, n, m, fmt)
    return p, sq.prep_export(p)


def assert_prep_matches(ex, op, rows=None):
    sel = slice(None) if rows is None else rows
    assert_bits_equal("mu", ex["mu"][sel], op.mu)
    assert_bits_equal("rstd", ex["rstd"][sel], op.rstd)
    assert_bits_equal("s_t", np.float32([ex["s_t"]]), np.float32([op.s_t]))
    assert_bits_equal("mask idx", ex["idx"][sel], op.idx)
    assert_bits_equal("S codes", ex["s_codes"][sel], op.s_codes)
    assert_bits_equal("S scales", ex["s_scales"][sel], op.s_scales)
    assert_bits_equal("R codes", ex["r_codes"][sel], op.r_codes)
    assert_bits_equal("R scales", ex["r_scales"][sel], op.r_scales)


def assert_weight_matches(wx, ow):
    assert_bits_equal("W codes", wx["codes"], ow.codes)
    assert_bits_equal("W scales (backbone view)", wx["scales"], ow.scales)
    assert_bits_equal("W scales (residual view)", wx["scales_residual"], ow.scales)
    assert_bits_equal("s_tW", np.float32([wx["s_tw"]]), np.float32([ow.s_tw]))


def assert_linear_close(got16: np.ndarray, want: np.ndarray, bound: np.ndarray, rel=1e-3):
    """Acceptance of the dual-path GEMM: |gpu - oracle| <= 1e-3 * sum|a||w| per
    output element (FP4 products are exact; only fp32 summation order and the
    final fp16 rounding differ), with an fp16 representation floor."""
    got = got16.astype(np.float64)
    err = np.abs(got - want)
    tol = rel * bound + FP16_FLOOR
    bad = err > tol
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"linear: {bad.sum()} elements out of tolerance; first {i}: gpu {got[i]} "
                             f"oracle {want[i]} bound {bound[i]}")
    return float((err / np.maximum(bound, 1e-30)).max()) if err.size else 0.0
