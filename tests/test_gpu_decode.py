"""GPU parity of the decode linear (1 to 16 token rows): the weight rows are
the block-scaled MMA's M side and the tokens its N side, each 128-row W tile
split over a cluster's K ranges. Checked against the oracle within
1e-3 * sum|a||w| per output element on every row: ragged n_out (a partial
last W tile), split factors that are not powers of two (48 W tiles), the
longest K of the dense layer set (56 K steps), both formats, every row
count class (1, odd, 16), fused segments with a bias; and that nothing is
written outside the output rows."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import assert_linear_close, cuda16, gpu_prepare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq():
    import sparsity_gemm_b200 as sq
    assert torch.cuda.is_available()
    sq.lib()
    return sq


CASES = [  # (m_tok, n_out, k, fmt, n, m)
    (1, 544, 1024, 0, 2, 4),     # 5 W tiles, the last one 32 rows
    (2, 544, 1024, 1, 2, 4),
    (5, 6144, 4096, 0, 2, 4),    # 48 tiles: a split of 6
    (16, 4096, 4096, 1, 2, 4),   # every token column of the MMA
    (7, 4096, 14336, 0, 2, 4),   # 56 K steps over clusters of 8
    (16, 256, 256, 0, 2, 4),     # one K step: no split
    (3, 128, 512, 1, 4, 8),
    (9, 14336, 4096, 0, 2, 4),   # 112 tiles: a split of 2
    (12, 992, 2048, 1, 3, 8),
    (2, 32, 512, 0, 2, 4),       # a weight smaller than one 128-row tile
]


@pytest.mark.parametrize("m_tok,n_out,k,fmt,n,m", CASES)
def test_decode_linear_within_tolerance(sq, m_tok, n_out, k, fmt, n, m):
    x = synth.activations_student(800 + m_tok, m_tok, k)
    w = synth.weights(801 + n_out, n_out, k)
    op = oracle.prepare(x, None, None, 1e-5, n, m, fmt)
    ow = oracle.quantize_weight(w, fmt)
    p, _ = gpu_prepare(x, None, None, 1e-5, n, m, fmt)
    out = sq.linear(p, sq.quantize_weight(cuda16(w), fmt)).cpu().numpy()
    want, bound = oracle.linear_prepared(op, ow)
    assert_linear_close(out, want, bound)
    assert sq.get_last_error() == sq.OK


@pytest.mark.parametrize("fmt,rows", [(0, [512, 128, 128]), (1, [512, 128, 128]), (0, [96, 160, 32])])
def test_decode_fused_segments_with_bias(sq, fmt, rows):
    """Fused segments with a bias; the last case puts segment boundaries
    inside 128-column W tiles (96, 256)."""
    k, m_tok = 2048, 4
    ws = [synth.weights(810 + i, r, k) * np.float16(1 + i) for i, r in enumerate(rows)]
    x = synth.activations_student(820, m_tok, k)
    b = synth.to_fp16(synth.normal(821, 0, sum(rows)) * 2.0)
    op = oracle.prepare(x, None, None, 1e-5, 2, 4, fmt)
    p, _ = gpu_prepare(x, None, None, 1e-5, 2, 4, fmt)
    fused = sq.quantize_weight_fused([cuda16(w) for w in ws], fmt)
    got = sq.linear(p, fused, bias=cuda16(b)).cpu().numpy()
    want, bound = oracle.linear_fused(op, oracle.quantize_weight_fused(ws, fmt), bias=b)
    assert_linear_close(got, want, bound)
    assert sq.get_last_error() == sq.OK


@pytest.mark.parametrize("m_tok", [1, 11, 16])
def test_decode_writes_only_its_rows(sq, m_tok):
    n_out, k = 640, 1024
    x = synth.activations_student(830 + m_tok, m_tok, k)
    w = synth.weights(831, n_out, k)
    p, _ = gpu_prepare(x, None, None, 1e-5, 2, 4, 0)
    buf = torch.full((m_tok + 2, n_out), 1234.0, dtype=torch.float16, device="cuda")
    out = buf[1:1 + m_tok]
    sq.linear(p, sq.quantize_weight(cuda16(w), 0), out=out)
    host = buf.cpu().numpy()
    assert np.all(host[0] == np.float16(1234.0)) and np.all(host[-1] == np.float16(1234.0))
    want, bound = oracle.linear_prepared(oracle.prepare(x, None, None, 1e-5, 2, 4, 0), oracle.quantize_weight(w, 0))
    assert_linear_close(host[1:1 + m_tok], want, bound)
    assert sq.get_last_error() == sq.OK
