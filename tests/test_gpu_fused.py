"""Fused projections (q/k/v, gate/up stacked into one weight) and the bias
epilogue on the GPU: the fused linear's columns equal the separate
linears' bit for bit (each segment keeps its own tensor scale, the K order
is the same), every segment's quantized payload equals the separately
quantized weight, and outputs with a bias match the oracle's fp64 value
plus the bias within the linear's tolerance. Covered: both formats, ragged
M over several tiles, segment boundaries that are not multiples of the
256-column tile, and the split-K launch (few rows)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import assert_bits_equal, assert_linear_close, cuda16, gpu_prepare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import sparsity_gemm_b200 as sq
    assert torch.cuda.is_available()
    sq.lib()
    yield


def _weights(seed, rows, k):
    return [synth.weights(seed + i, r, k) * np.float16(1 + i) for i, r in enumerate(rows)]


def _values_equal(a, b):
    """fp16 arrays equal as values (+0 == -0), NaN-free."""
    return np.array_equal(a.astype(np.float32), b.astype(np.float32))


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("m_tok,rows,k", [(300, [512, 160, 96], 512), (8, [256, 128, 128], 1024),
                                          (130, [224, 288], 768)])
def test_fused_equals_separate_linears(fmt, m_tok, rows, k):
    import sparsity_gemm_b200 as sq
    ws = _weights(400 + m_tok, rows, k)
    x = synth.activations_student(410 + m_tok, m_tok, k)
    p, _ = gpu_prepare(x, None, None, 1e-5, 2, 4, fmt)
    fused = sq.quantize_weight_fused([cuda16(w) for w in ws], fmt)
    assert fused.desc.segments == len(rows) and list(fused.desc.seg_end)[:len(rows)] == list(np.cumsum(rows))
    got = sq.linear(p, fused).cpu().numpy()
    sep_scales = []
    col = 0
    fx = sq.weight_export(fused)
    for w, r in zip(ws, rows):
        qw = sq.quantize_weight(cuda16(w), fmt)
        want = sq.linear(p, qw).cpu().numpy()
        assert_bits_equal(f"columns {col}..{col + r}", got[:, col:col + r].view(np.uint16), want.view(np.uint16))
        wx = sq.weight_export(qw)
        assert_bits_equal("segment codes", fx["codes"][col:col + r], wx["codes"])
        assert_bits_equal("segment scales", fx["scales"][col:col + r], wx["scales"])
        sep_scales.append(wx["s_tw"])
        col += r
    assert_bits_equal("segment tensor scales", sq.weight_tensor_scales(fused), np.float32(sep_scales))
    assert sq.get_last_error() == sq.OK


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("m_tok,rows,k", [(200, [256, 64, 64], 512), (5, [128, 96], 256)])
def test_fused_with_bias_against_oracle(fmt, m_tok, rows, k):
    import sparsity_gemm_b200 as sq
    ws = _weights(420 + m_tok, rows, k)
    x = synth.activations_student(430 + m_tok, m_tok, k)
    op = oracle.prepare(x, None, None, 1e-5, 2, 4, fmt)
    p, _ = gpu_prepare(x, None, None, 1e-5, 2, 4, fmt)
    b = synth.to_fp16(synth.normal(440 + m_tok, 0, sum(rows)) * 2.0)
    fused = sq.quantize_weight_fused([cuda16(w) for w in ws], fmt)
    got = sq.linear(p, fused, bias=cuda16(b)).cpu().numpy()
    want, bound = oracle.linear_fused(op, oracle.quantize_weight_fused(ws, fmt), bias=b)
    assert_linear_close(got, want, bound)
    # a zero bias changes no value
    plain = sq.linear(p, fused).cpu().numpy()
    zero = sq.linear(p, fused, bias=torch.zeros(sum(rows), dtype=torch.float16, device="cuda")).cpu().numpy()
    assert _values_equal(plain, zero)
    assert sq.get_last_error() == sq.OK


def test_bias_on_a_plain_weight_and_split_k():
    """Bias with one segment, at a tile-filling size and at a few-row size
    whose launch splits K across a cluster."""
    import sparsity_gemm_b200 as sq
    for m_tok, n_out, k in [(257, 512, 512), (3, 256, 2048)]:
        w = synth.weights(450 + m_tok, n_out, k)
        x = synth.activations_student(451 + m_tok, m_tok, k)
        op = oracle.prepare(x, None, None, 1e-5, 2, 4, 0)
        p, _ = gpu_prepare(x, None, None, 1e-5, 2, 4, 0)
        b = synth.to_fp16(synth.normal(452 + m_tok, 0, n_out))
        qw = sq.quantize_weight(cuda16(w), 0)
        got = sq.linear(p, qw, bias=cuda16(b)).cpu().numpy()
        want, bound = oracle.linear_fused(op, [oracle.quantize_weight(w, 0)], bias=b)
        assert_linear_close(got, want, bound)
    assert sq.get_last_error() == sq.OK
