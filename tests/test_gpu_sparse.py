"""GPU parity of the pair-wise 4:8 sparse-backbone mode (sharq_prepare_sparse,
sharq_quantize_weight_sparse, and sharq_linear through tcgen05.mma.sp)
against the oracle: the mask, the K-compacted backbone codes (exported in
canonical form), every scale and the statistics bit for bit; the linear
within 1e-3 * sum|a||w| per output element."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import assert_bits_equal, assert_linear_close, assert_prep_matches, cuda16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq():
    import sparsity_gemm_b200 as sq
    assert torch.cuda.is_available()
    sq.lib()
    return sq


PREP_CASES = [  # (m_tok, k, fmt, affine, norm)
    (300, 1024, 0, False, "layer"),
    (129, 2048, 1, True, "layer"),
    (200, 4096, 0, True, "rms"),
    (64, 4096, 1, False, "rms"),
    (1, 512, 0, False, "layer"),
    (37, 256, 0, True, "layer"),
]


def _ln(affine, norm, k, seed):
    if not affine:
        return None, None
    g, b = synth.ln_params(seed, k)
    return g, (b if norm == "layer" else None)


@pytest.mark.parametrize("m_tok,k,fmt,affine,norm", PREP_CASES)
def test_sparse_prep_bit_exact(sq, m_tok, k, fmt, affine, norm):
    x = synth.activations_student(100 + m_tok, m_tok, k)
    g, b = _ln(affine, norm, k, 7)
    p = sq.prepare_sparse(cuda16(x), None if g is None else cuda16(g), None if b is None else cuda16(b), 1e-5, fmt,
                          norm=norm)
    ex = sq.prep_export(p)
    op = oracle.prepare_sparse(x, g, b, 1e-5, fmt, norm=norm)
    assert_prep_matches(ex, op)
    assert sq.get_last_error() == sq.OK


def test_sparse_prep_no_rows(sq):
    x = torch.zeros((0, 512), dtype=torch.float16, device="cuda")
    p = sq.prepare_sparse(x, None, None, 1e-5, 0)
    assert float(sq.prep_export(p)["s_t"]) == 1.0
    assert sq.get_last_error() == sq.OK


@pytest.mark.parametrize("fmt", [0, 1])
def test_sparse_weight_bit_exact(sq, fmt):
    w = synth.weights(200 + fmt, 544, 1024)
    qw = sq.quantize_weight_sparse(cuda16(w), fmt)
    wx = sq.weight_export(qw)
    ow = oracle.quantize_weight_sparse(w, fmt)
    assert_bits_equal("W codes", wx["codes"], ow.codes)
    assert_bits_equal("W scales (backbone view)", wx["scales"], ow.scales)
    assert_bits_equal("W scales (residual view)", wx["scales_residual"], np.repeat(ow.scales, 2, axis=1))
    assert_bits_equal("s_tW", np.float32([wx["s_tw"]]), np.float32([ow.s_tw]))


LINEAR_CASES = [  # (m_tok, n_out, k, fmt): ragged m and n, 1 .. 8 K tiles, split-K for few tiles
    (300, 544, 1024, 0),
    (300, 544, 1024, 1),
    (129, 256, 2048, 0),
    (200, 288, 256, 0),
    (8, 1024, 4096, 0),
    (1, 512, 2048, 1),
    (1000, 4096, 4096, 0),
]


@pytest.mark.parametrize("m_tok,n_out,k,fmt", LINEAR_CASES)
def test_sparse_linear_within_tolerance(sq, m_tok, n_out, k, fmt):
    x = synth.activations_student(300 + m_tok, m_tok, k)
    w = synth.weights(301 + n_out, n_out, k)
    p = sq.prepare_sparse(cuda16(x), None, None, 1e-5, fmt)
    qw = sq.quantize_weight_sparse(cuda16(w), fmt)
    out = sq.linear(p, qw).cpu().numpy()
    rows = np.unique(np.r_[np.arange(min(m_tok, 40)), m_tok - 1,
                           np.random.default_rng(3).choice(m_tok, size=min(24, m_tok), replace=False)])
    op = oracle.prepare_sparse(x[rows], None, None, 1e-5, fmt, s_t=np.float32(sq.prep_export(p)["s_t"]))
    ow = oracle.quantize_weight_sparse(w, fmt)
    want, bound = oracle.linear_sparse(op, ow)
    assert_linear_close(out[rows], want, bound)
    assert sq.get_last_error() == sq.OK


def test_sparse_modes_do_not_mix(sq):
    x = cuda16(synth.activations_student(400, 64, 512))
    w = cuda16(synth.weights(401, 256, 512))
    ps, pd = sq.prepare_sparse(x, None, None, 1e-5, 0), sq.prepare(x, None, None, 1e-5, 2, 4, 0)
    ws, wd = sq.quantize_weight_sparse(w, 0), sq.quantize_weight(w, 0)
    for p, q in [(ps, wd), (pd, ws)]:
        with pytest.raises(sq.SharqError) as e:
            sq.linear(p, q)
        assert e.value.status == sq.ERR_INVALID_ARG
    with pytest.raises(sq.SharqError) as e:
        sq.linear(ps, ws, bias=torch.zeros(256, dtype=torch.float16, device="cuda"))
    assert e.value.status == sq.ERR_UNSUPPORTED
    assert sq.get_last_error() == sq.OK
