"""Pins for the oracle's fused projections and bias (segments quantized on
their own and placed side by side; the bias added after the scaled
accumulator):

- segments whose amax agree quantize exactly like the stacked weight, so the
  fused linear is the linear of the stacked weight;
- a segment that is another scaled by 2^-2 keeps its own tensor scale
  (2^-2 times the other's) and the same codes, which a quantization of the
  stacked weight (one shared amax) would not give;
- on an all-zero weight the output is the bias itself;
- fused output plus bias against an independent dequantization (ml_dtypes
  codecs) of the prepared activation and of each segment's weight.
"""
import ml_dtypes
import numpy as np

import synth


def _deq(codes, scales, fmt):
    blk = 16 if fmt == 0 else 32
    v = (codes & 0xF).astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    t = ml_dtypes.float8_e4m3fn if fmt == 0 else ml_dtypes.float8_e8m0fnu
    return v * np.repeat(scales.view(t).astype(np.float64), blk, axis=1)


def test_equal_amax_segments_are_the_stacked_weight(orc):
    k = 256
    w1 = synth.weights(90, 64, k)
    w2 = synth.weights(91, 96, k)
    i1 = np.unravel_index(np.argmax(np.abs(w1.astype(np.float32))), w1.shape)
    w2[3, 17] = w1[i1]  # the same amax in both segments
    assert np.abs(w2.astype(np.float32)).max() == np.abs(w1.astype(np.float32)).max()
    for fmt in (0, 1):
        q1, q2 = orc.quantize_weight_fused([w1, w2], fmt)
        qs = orc.quantize_weight(np.concatenate([w1, w2]), fmt)
        assert q1.s_tw == q2.s_tw == qs.s_tw
        assert np.array_equal(np.concatenate([q1.codes, q2.codes]), qs.codes)
        assert np.array_equal(np.concatenate([q1.scales, q2.scales]), qs.scales)
        x = synth.activations_student(92, 5, k)
        p = orc.prepare(x, None, None, 1e-5, 2, 4, fmt)
        got, _ = orc.linear_fused(p, [q1, q2])
        want, _ = orc.linear_prepared(p, qs)
        assert np.array_equal(got, want)


def test_each_segment_keeps_its_own_tensor_scale(orc):
    k = 512
    w1 = synth.weights(93, 64, k)
    w1[np.abs(w1.astype(np.float32)) < 2.0 ** -10] = np.float16(2.0 ** -10)  # no fp16 subnormal after / 4
    w2 = (w1.astype(np.float32) / 4).astype(np.float16)
    assert np.array_equal(w2.astype(np.float32) * 4, w1.astype(np.float32))  # exact
    q1, q2 = orc.quantize_weight_fused([w1, w2], 0)
    assert q2.s_tw == np.float32(q1.s_tw / 4)
    assert np.array_equal(q1.codes, q2.codes) and np.array_equal(q1.scales, q2.scales)
    stacked = orc.quantize_weight(np.concatenate([w1, w2]), 0)
    assert not np.array_equal(stacked.codes[64:], q2.codes) or not np.array_equal(stacked.scales[64:], q2.scales)
    x = synth.activations_student(94, 7, k)
    p = orc.prepare(x, None, None, 1e-5, 2, 4, 0)
    out, _ = orc.linear_fused(p, [q1, q2])
    assert np.array_equal(out[:, 64:] * 4, out[:, :64])


def test_zero_weight_gives_the_bias(orc):
    k, n = 256, 64
    x = synth.activations_student(95, 4, k)
    p = orc.prepare(x, None, None, 1e-5, 2, 4, 0)
    qws = orc.quantize_weight_fused([np.zeros((32, k), np.float16), np.zeros((32, k), np.float16)], 0)
    b = synth.to_fp16(np.linspace(-3.0, 5.0, n))
    out, bound = orc.linear_fused(p, qws, bias=b)
    assert np.array_equal(out, np.broadcast_to(b.astype(np.float64), out.shape))
    assert np.array_equal(bound, np.broadcast_to(np.abs(b.astype(np.float64)), out.shape))


def test_fused_with_bias_against_independent_dequantization(orc):
    k = 256
    for fmt in (0, 1):
        ws = [synth.weights(96, 64, k), synth.weights(97, 32, k) * np.float16(3), synth.weights(98, 32, k)]
        qws = orc.quantize_weight_fused(ws, fmt)
        x = synth.activations_student(99, 6, k)
        p = orc.prepare(x, None, None, 1e-5, 2, 4, fmt)
        b = synth.to_fp16(synth.normal(100, 0, 128))
        out, _ = orc.linear_fused(p, qws, bias=b)
        a = (_deq(p.s_codes, p.s_scales, fmt) + _deq(p.r_codes, p.r_scales, fmt)) * float(p.s_t)
        col = 0
        for q in qws:
            wv = _deq(q.codes, q.scales, fmt) * float(q.s_tw)
            want = a @ wv.T + b[col:col + q.codes.shape[0]].astype(np.float64)
            assert np.allclose(out[:, col:col + q.codes.shape[0]], want, rtol=1e-12, atol=1e-12)
            col += q.codes.shape[0]
