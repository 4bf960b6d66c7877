"""Pins for the oracle's pair-wise 4:8 sparse-backbone mode.

The mode's mask is checked against a brute-force restatement (a pair is kept
iff fewer than two pairs beat it) on random and constructed-tie groups; the
backbone's blocks of 32 (NVFP4) / 64 (MXFP4) logical values against the
format's plain quantization of the K-compacted kept values (the same block
of 16 / 32 stored values); scales and codes against an independent codec
library; the reconstruction invariant deq(Q(S)) + R == X_ln bitwise; and the
GEMM with per-array block lengths against a library matmul of operands
dequantized with that library, and against the default-mode GEMM when the
block lengths are the format's own."""
import itertools

import ml_dtypes
import numpy as np
import pytest

import synth

SPARSE_BLK = {0: 32, 1: 64}
BLK = {0: 16, 1: 32}


def _brute_pairs(v):
    """Kept pairs of one group of 8: pair j is kept iff fewer than two pairs
    beat it, where pair i beats pair j if its larger magnitude is larger, or
    equal with i < j."""
    key = [max(abs(float(v[2 * j])), abs(float(v[2 * j + 1]))) for j in range(4)]
    kept = []
    for j in range(4):
        beaten_by = sum(1 for i in range(4) if i != j and (key[i] > key[j] or (key[i] == key[j] and i < j)))
        if beaten_by < 2:
            kept.append(j)
    return kept


def _groups_with_ties(rng, count):
    vals = np.float32([0.0, -0.0, 0.5, -0.5, 1.0, 3.0, -3.0, 7.25])
    return rng.choice(vals, size=(count, 8)).astype(np.float32)


def test_pair_mask_matches_brute_force(orc):
    rng = np.random.default_rng(3)
    rows = np.concatenate([rng.standard_normal((64, 8)).astype(np.float32),
                           _groups_with_ties(rng, 256),
                           np.zeros((1, 8), np.float32),
                           np.float32([[-0.0, 0.0, 0.0, -0.0, 0.0, 0.0, -0.0, -0.0]]),
                           np.float32([[1, 1, 1, 1, 1, 1, 1, 1]]),
                           np.float32([[0, 5, 5, 0, 0, 0, 0, 5]])])
    x = rows.reshape(-1, 64) if rows.shape[0] % 8 == 0 else np.concatenate(
        [rows, np.zeros((8 - rows.shape[0] % 8, 8), np.float32)]).reshape(-1, 64)
    idx, keep = orc.mask_pairs48(x)
    g = x.reshape(-1, 8)
    gi = idx.reshape(-1, 4)
    gk = keep.reshape(-1, 8)
    for t in range(g.shape[0]):
        pairs = _brute_pairs(g[t])
        assert len(pairs) == 2
        want = [2 * pairs[0], 2 * pairs[0] + 1, 2 * pairs[1], 2 * pairs[1] + 1]
        assert list(gi[t]) == want, (g[t], gi[t], want)
        assert [int(b) for b in gk[t]] == [1 if i // 2 in pairs else 0 for i in range(8)]


def test_pair_mask_structure(orc):
    x = synth.activations_student(5, 16, 512).astype(np.float32)
    idx, keep = orc.mask_pairs48(x)
    g = np.abs(x.reshape(-1, 8))
    k = keep.reshape(-1, 8)
    assert np.all(k.sum(1) == 4)
    assert np.all(k[:, 0::2] == k[:, 1::2])  # whole adjacent pairs
    key = np.maximum(g[:, 0::2], g[:, 1::2])
    kp = k[:, 0::2] == 1
    assert np.all(np.where(kp, key, np.inf).min(1) >= np.where(~kp, key, -np.inf).max(1))
    # the group's largest magnitude is always kept
    assert np.all(k[np.arange(len(g)), g.argmax(1)] == 1)


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("affine", [False, True])
def test_sparse_reconstruction_is_exact(orc, fmt, affine):
    x = synth.activations_student(11 + fmt, 10, 512)
    g, b = synth.ln_params(4, 512) if affine else (None, None)
    p = orc.prepare_sparse(x, g, b, 1e-5, fmt)
    rebuilt = (p.deq_s + p.r).astype(np.float32)
    assert np.array_equal(rebuilt.view(np.uint32), p.x_ln.view(np.uint32))
    assert np.array_equal(p.r[p.keep == 0], p.x_ln[p.keep == 0])
    assert np.all(p.s_codes[p.keep == 0] == 0)


@pytest.mark.parametrize("fmt", [0, 1])
def test_backbone_blocks_are_the_format_on_compacted_values(orc, fmt):
    """A backbone block of 32 (64) logical values holds 16 (32) kept values;
    its scale and codes are the format's plain quantization of those values
    taken in order (the K-compacted operand the sparse MMA reads)."""
    x = synth.activations_student(21 + fmt, 9, 1024)
    p = orc.prepare_sparse(x, None, None, 1e-5, fmt)
    rows, k = x.shape
    kept_vals = p.s[p.keep == 1].reshape(rows, k // 2)
    kept_codes = p.s_codes[p.keep == 1].reshape(rows, k // 2)
    codes, scales = orc.quantize(kept_vals, fmt, p.s_t)
    assert np.array_equal(scales, p.s_scales)
    assert np.array_equal(codes, kept_codes)


@pytest.mark.parametrize("fmt", [0, 1])
def test_sparse_scales_and_codes_with_library_codecs(orc, fmt):
    x = synth.activations_student(31 + fmt, 8, 512)
    p = orc.prepare_sparse(x, None, None, 1e-5, fmt)
    rows, k = x.shape
    for vals, codes, scales, blk in [(p.s, p.s_codes, p.s_scales, SPARSE_BLK[fmt]),
                                     (p.r, p.r_codes, p.r_scales, BLK[fmt])]:
        a = np.abs(vals).reshape(rows, k // blk, blk).max(-1)
        if fmt == 0:
            u = a / (np.float32(6.0) * p.s_t)
            want = np.minimum(u, np.float32(448)).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
            d = scales.view(ml_dtypes.float8_e4m3fn).astype(np.float32) * p.s_t
        else:
            e = np.frexp(a.astype(np.float64))[1] - 3
            want = np.where(a == 0, 0, np.clip(e, -127, 127) + 127).astype(np.uint8)
            d = scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float32)
        assert np.array_equal(scales, want)
        d = np.repeat(d, blk, axis=1)
        nz = d != 0
        q = (vals[nz] / d[nz]).astype(np.float32)
        assert np.array_equal(codes[nz], q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF)


def test_two_pairs_per_group_is_plain_quantization_of_the_backbone(orc):
    """Rows whose groups hold non-zeros in two pairs only: the backbone is
    X_ln itself and R its quantization error (blocks of 32)."""
    rng = np.random.default_rng(9)
    rows, k = 6, 256
    v = np.zeros((rows, k // 8, 8), np.float32)
    for r, g in itertools.product(range(rows), range(k // 8)):
        i, j = sorted(rng.choice(4, 2, replace=False))
        v[r, g, 2 * i:2 * i + 2] = rng.standard_normal(2)
        v[r, g, 2 * j:2 * j + 2] = rng.standard_normal(2)
    v = v.reshape(rows, k)
    idx, keep = orc.mask_pairs48(v)
    assert np.array_equal(keep == 1, v != 0)
    codes, scales = orc.quantize_blk(v, 0, 32, 0.01)
    codes16, scales16 = orc.quantize(v[keep == 1].reshape(rows, k // 2), 0, 0.01)
    assert np.array_equal(scales, scales16) and np.array_equal(codes[keep == 1].reshape(rows, -1), codes16)


@pytest.mark.parametrize("fmt", [0, 1])
def test_sparse_weights_and_residual_view(orc, fmt):
    """Weights of the pair-wise mode: blocks of 32 (64), scales and codes
    from the library codecs; repeating every scale twice gives the residual
    path's view at the format's own block length with the same values."""
    w = synth.weights(41, 64, 512)
    qw = orc.quantize_weight_sparse(w, fmt)
    blk = SPARSE_BLK[fmt]
    wf = w.astype(np.float32)
    a = np.abs(wf).reshape(64, 512 // blk, blk).max(-1)
    if fmt == 0:
        assert qw.s_tw == np.float32(np.abs(wf).max()) / np.float32(2688)
        want = np.minimum(a / (np.float32(6) * qw.s_tw), np.float32(448)).astype(ml_dtypes.float8_e4m3fn)
        assert np.array_equal(qw.scales, want.view(np.uint8))
    else:
        e = np.frexp(a.astype(np.float64))[1] - 3
        assert np.array_equal(qw.scales, np.where(a == 0, 0, np.clip(e, -127, 127) + 127).astype(np.uint8))
    dense_view = np.repeat(qw.scales, 2, axis=1)
    out_view, _ = orc.linear(np.zeros((1, 512), np.uint8), np.zeros((1, 512 // BLK[fmt]), np.uint8),
                             np.full((1, 512), 2, np.uint8), np.full((1, 512 // BLK[fmt]), 56 if fmt == 0 else 127,
                                                                      np.uint8),
                             1.0, qw.codes, dense_view, qw.s_tw, fmt)
    out_blk, _ = orc.linear_blk(np.zeros((1, 512), np.uint8), np.zeros((1, 512 // blk), np.uint8), blk,
                                np.full((1, 512), 2, np.uint8),
                                np.full((1, 512 // BLK[fmt]), 56 if fmt == 0 else 127, np.uint8), BLK[fmt],
                                1.0, qw.codes, qw.scales, blk, qw.s_tw, fmt)
    assert np.array_equal(out_view, out_blk)


def _deq(codes, scales, fmt, blk):
    v = (codes & 0xF).astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    t = ml_dtypes.float8_e4m3fn if fmt == 0 else ml_dtypes.float8_e8m0fnu
    return v * np.repeat(scales.view(t).astype(np.float64), blk, axis=1)


@pytest.mark.parametrize("fmt", [0, 1])
def test_sparse_linear_matches_library_matmul(orc, fmt):
    x = synth.activations_student(51 + fmt, 7, 512)
    w = synth.weights(52, 40, 512)
    p = orc.prepare_sparse(x, None, None, 1e-5, fmt)
    qw = orc.quantize_weight_sparse(w, fmt)
    out, bound = orc.linear_sparse(p, qw)
    sb, rb = SPARSE_BLK[fmt], BLK[fmt]
    a_s, a_r = _deq(p.s_codes, p.s_scales, fmt, sb), _deq(p.r_codes, p.r_scales, fmt, rb)
    b = _deq(qw.codes, qw.scales, fmt, sb)
    ts = float(p.s_t) * float(qw.s_tw)
    ref = ts * ((a_s + a_r) @ b.T)
    mag = ts * ((np.abs(a_s) + np.abs(a_r)) @ np.abs(b).T)
    assert np.allclose(out, ref, rtol=0, atol=1e-12 * mag.max())
    assert np.allclose(bound, mag, rtol=1e-12)


def test_linear_blk_with_the_formats_blocks_is_the_default_linear(orc):
    x = synth.activations_student(61, 5, 256)
    w = synth.weights(62, 24, 256)
    for fmt in (0, 1):
        p = orc.prepare(x, None, None, 1e-5, 2, 4, fmt)
        qw = orc.quantize_weight(w, fmt)
        a, ab = orc.linear_prepared(p, qw)
        b, bb = orc.linear_blk(p.s_codes, p.s_scales, BLK[fmt], p.r_codes, p.r_scales, BLK[fmt], p.s_t,
                               qw.codes, qw.scales, BLK[fmt], qw.s_tw, fmt)
        assert np.array_equal(a, b) and np.array_equal(ab, bb)
