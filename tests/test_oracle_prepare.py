"""Pins for the oracle's preparation operator: the invariants the abstract
fixes (the residual is taken against the quantized backbone, so
deq(Q(S)) + R == X_ln exactly in fp32), the n = m special case (plain block
quantization), exactly representable inputs (zero residual), and the scale
and code values re-derived with an independent codec library."""
import ml_dtypes
import numpy as np
import pytest

import synth

CASES = [(0, 2, 4), (0, 4, 8), (0, 1, 2), (1, 2, 4), (1, 4, 8), (0, 1, 4), (1, 8, 16)]


def _x(seed, rows=12, k=512):
    return synth.activations_student(seed, rows, k)


def _code_values(codes):
    return (codes & 0xF).astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float32)


def _scale_values(scales, fmt):
    t = ml_dtypes.float8_e4m3fn if fmt == 0 else ml_dtypes.float8_e8m0fnu
    return scales.view(t).astype(np.float32)


@pytest.mark.parametrize("fmt,n,m", CASES)
@pytest.mark.parametrize("affine", [False, True])
def test_reconstruction_is_exact(orc, fmt, n, m, affine):
    x = _x(fmt * 10 + n + m)
    g, b = synth.ln_params(4, x.shape[1]) if affine else (None, None)
    p = orc.prepare(x, g, b, 1e-5, n, m, fmt)
    rebuilt = (p.deq_s + p.r).astype(np.float32)  # float32 + float32, RN
    assert np.array_equal(rebuilt.view(np.uint32), p.x_ln.view(np.uint32))


@pytest.mark.parametrize("fmt,n,m", CASES)
def test_backbone_structure_and_scales(orc, fmt, n, m):
    x = _x(20 + fmt, rows=8, k=256)
    p = orc.prepare(x, None, None, 1e-5, n, m, fmt)
    blk = 16 if fmt == 0 else 32
    rows, k = x.shape
    # S is X_ln on the kept positions and +0 elsewhere; so are its codes
    assert np.array_equal(p.s, np.where(p.keep == 1, p.x_ln, np.float32(0)))
    assert np.all(p.s_codes[p.keep == 0] == 0)
    # tensor scale: amax(S) == amax(X_ln) when n >= 1, s_t = RN32(amax / 2688)
    amax = np.abs(p.x_ln).max()
    assert np.abs(p.s).max() == amax
    if fmt == 0:
        assert p.s_t == np.float32(amax) / np.float32(2688.0)
    else:
        assert p.s_t == 1.0
    # block scales re-derived with the library codecs
    for vals, scales in [(p.s, p.s_scales), (p.r, p.r_scales)]:
        a = np.abs(vals).reshape(rows, k // blk, blk).max(-1)
        if fmt == 0:
            u = a / (np.float32(6.0) * p.s_t)
            want = np.minimum(u, np.float32(448)).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
        else:
            e = np.frexp(a.astype(np.float64))[1] - 3
            want = np.where(a == 0, 0, np.clip(e, -127, 127) + 127).astype(np.uint8)
        assert np.array_equal(scales, want)
    # dequantized backbone = code value * RN32(scale * s_t), with library decoders
    d = _scale_values(p.s_scales, fmt)
    if fmt == 0:
        d = d * p.s_t
    d = np.repeat(d, blk, axis=1)
    deq = _code_values(p.s_codes) * d
    assert np.array_equal(np.where(p.keep == 1, deq, np.float32(0)), p.deq_s)
    # codes are the library's E2M1 of v / d, off the zero-step blocks
    for vals, codes, scales in [(p.s, p.s_codes, p.s_scales), (p.r, p.r_codes, p.r_scales)]:
        dd = _scale_values(scales, fmt)
        if fmt == 0:
            dd = dd * p.s_t
        dd = np.repeat(dd, blk, axis=1)
        nz = dd != 0
        q = (vals[nz] / dd[nz]).astype(np.float32)
        want = q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
        assert np.array_equal(codes[nz], want)
        assert np.all(codes[~nz] == 0)


@pytest.mark.parametrize("fmt", [0, 1])
def test_residual_bounded_by_amax(orc, fmt):
    p = orc.prepare(_x(31), None, None, 1e-5, 2, 4, fmt)
    assert np.abs(p.r).max() <= np.abs(p.x_ln).max()
    kept = p.keep == 1
    assert np.all(np.abs(p.r[kept]) <= np.abs(p.x_ln[kept]))  # deq has x's sign, |deq| <= 2|x|
    assert np.array_equal(p.r[~kept], p.x_ln[~kept])


@pytest.mark.parametrize("fmt", [0, 1])
def test_n_equals_m_is_plain_quantization(orc, fmt):
    x = _x(40 + fmt)
    p = orc.prepare(x, None, None, 1e-5, 4, 4, fmt)
    assert np.all(p.keep == 1)
    codes, scales = orc.quantize(p.x_ln, fmt, p.s_t)
    assert np.array_equal(codes, p.s_codes) and np.array_equal(scales, p.s_scales)
    # R is then the pure quantization error of X_ln
    err = p.x_ln - p.deq_s
    assert np.array_equal(err, p.r)


def test_exactly_representable_values_quantize_without_error(orc):
    grid = np.float32([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    rng = np.random.default_rng(8)
    # MXFP4: block values grid * 2^e with one element at 6 * 2^e
    for e in [-20, -1, 0, 3, 40]:
        v = (rng.choice(grid, 32) * rng.choice([-1, 1], 32)).astype(np.float32)
        v[5] = 6.0
        v = (v * np.float32(2.0 ** e))[None, :]
        codes, scales = orc.quantize(v, 1, 1.0)
        assert scales[0, 0] == e + 127
        assert np.array_equal(_code_values(codes) * np.float32(2.0 ** e), v)
    # NVFP4: s_t a power of two, scale value exact in UE4M3, amax = 6 * d
    for s_t, sb in [(2.0 ** -4, 1.5), (1.0, 0.25), (2.0 ** 3, 448.0), (2.0 ** -10, 2.0 ** -9)]:
        d = np.float32(sb * s_t)
        v = (rng.choice(grid, 16) * rng.choice([-1, 1], 16)).astype(np.float32)
        v[0] = -6.0
        v = (v * d)[None, :]
        codes, scales = orc.quantize(v, 0, s_t)
        assert np.float32(scales[0].view(ml_dtypes.float8_e4m3fn)[0]) == np.float32(sb)
        assert np.array_equal(_code_values(codes) * d, v)


@pytest.mark.parametrize("fmt", [0, 1])
def test_sharq_error_below_plain_fp4(orc, fmt):
    """Quality sanity on the 16x256 single-linear workload: the dual path's
    output error against the unquantized product is below plain FP4's."""
    x = synth.activations_gaussian(0, 16, 256, 4, 50.0)
    w = synth.weights(1, 256, 256)
    qw = orc.quantize_weight(w, fmt)
    p = orc.prepare(x, None, None, 1e-5, 2, 4, fmt)
    ref = p.x_ln.astype(np.float64) @ qw.w_f32.T.astype(np.float64)
    out, _ = orc.linear_prepared(p, qw)
    plain = orc.prepare(x, None, None, 1e-5, 4, 4, fmt)
    out_plain, _ = orc.linear(plain.s_codes, plain.s_scales, np.zeros_like(plain.r_codes),
                              plain.r_scales, plain.s_t, qw.codes, qw.scales, qw.s_tw, fmt)
    e_sharq = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    e_plain = np.linalg.norm(out_plain - ref) / np.linalg.norm(ref)
    assert e_sharq < e_plain
