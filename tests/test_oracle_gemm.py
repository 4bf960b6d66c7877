"""Pins for the oracle's dual-path GEMM: a library matmul on matrices
dequantized with an independent codec library, one-hot weight rows that
reduce the GEMM to dequantization, linearity in the two paths, and the
tolerance scale bounding the output."""
import ml_dtypes
import numpy as np
import pytest

import synth


def _deq(codes, scales, fmt):
    blk = 16 if fmt == 0 else 32
    v = (codes & 0xF).astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    t = ml_dtypes.float8_e4m3fn if fmt == 0 else ml_dtypes.float8_e8m0fnu
    s = np.repeat(scales.view(t).astype(np.float64), blk, axis=1)
    return v * s


@pytest.mark.parametrize("fmt,n,m", [(0, 2, 4), (1, 2, 4), (0, 4, 8), (1, 1, 2)])
def test_linear_matches_library_matmul(orc, fmt, n, m):
    x = synth.activations_student(50 + fmt, 7, 256)
    w = synth.weights(51, 40, 256)
    p = orc.prepare(x, None, None, 1e-5, n, m, fmt)
    qw = orc.quantize_weight(w, fmt)
    out, bound = orc.linear_prepared(p, qw)
    a = _deq(p.s_codes, p.s_scales, fmt) + _deq(p.r_codes, p.r_scales, fmt)
    b = _deq(qw.codes, qw.scales, fmt)
    ref = float(p.s_t) * float(qw.s_tw) * (a @ b.T)
    mag = float(p.s_t) * float(qw.s_tw) * (np.abs(_deq(p.s_codes, p.s_scales, fmt)) +
                                           np.abs(_deq(p.r_codes, p.r_scales, fmt))) @ np.abs(b).T
    assert np.allclose(out, ref, rtol=0, atol=1e-12 * mag.max())
    assert np.allclose(bound, mag, rtol=1e-12)
    assert np.all(np.abs(out) <= bound * (1 + 1e-12))


def test_one_hot_weights_reduce_to_dequantization(orc):
    fmt = 0
    x = synth.activations_student(60, 5, 128)
    p = orc.prepare(x, None, None, 1e-5, 2, 4, fmt)
    cols = np.array([0, 17, 64, 127, 3])
    w_codes = np.zeros((len(cols), 128), np.uint8)
    w_scales = np.zeros((len(cols), 128 // 16), np.uint8)
    for j, c in enumerate(cols):
        w_codes[j, c] = 2                # E2M1 1.0
        w_scales[j, c // 16] = 56        # UE4M3 1.0
    out, _ = orc.linear(p.s_codes, p.s_scales, p.r_codes, p.r_scales, p.s_t,
                        w_codes, w_scales, 1.0, fmt)
    a = (_deq(p.s_codes, p.s_scales, fmt) + _deq(p.r_codes, p.r_scales, fmt)) * float(p.s_t)
    assert np.array_equal(out, a[:, cols])


def test_linear_is_the_sum_of_its_paths(orc):
    fmt = 0
    x = synth.activations_student(61, 6, 256)
    w = synth.weights(62, 32, 256)
    p = orc.prepare(x, None, None, 1e-5, 2, 4, fmt)
    qw = orc.quantize_weight(w, fmt)
    z = np.zeros_like(p.s_codes)
    both, _ = orc.linear(p.s_codes, p.s_scales, p.r_codes, p.r_scales, p.s_t, qw.codes, qw.scales, qw.s_tw, fmt)
    s_only, _ = orc.linear(p.s_codes, p.s_scales, z, p.r_scales, p.s_t, qw.codes, qw.scales, qw.s_tw, fmt)
    r_only, _ = orc.linear(z, p.s_scales, p.r_codes, p.r_scales, p.s_t, qw.codes, qw.scales, qw.s_tw, fmt)
    assert np.allclose(both, s_only + r_only, rtol=1e-12, atol=1e-300)


def test_weight_quantization_scale(orc):
    w = synth.weights(63, 64, 256)
    qw = orc.quantize_weight(w, 0)
    assert qw.s_tw == np.float32(np.abs(w.astype(np.float32)).max()) / np.float32(2688)
    assert np.array_equal(qw.w_f32, w.astype(np.float32))
    qm = orc.quantize_weight(w, 1)
    assert qm.s_tw == 1.0
