"""GPU parity of sharq_prepare_add: the residual add x = RN16(h + d) fused with
the preparation operator's statistics pass. x is compared with the oracle's
binary16 add bit for bit, the prepared outputs with the oracle's preparation
of that x bit for bit, and with sharq_prepare on the stored x (the unfused
path) bit for bit; in-place (x_out = h) gives the same."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import assert_bits_equal, assert_prep_matches, cuda16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq():
    import sparsity_gemm_b200 as sq
    assert torch.cuda.is_available()
    sq.lib()
    return sq


CASES = [  # (m_tok, k, fmt, n, m, affine, norm)
    (300, 1024, 0, 2, 4, False, "layer"),   # exact integer sums
    (129, 4096, 1, 4, 8, True, "layer"),    # certified sums, the affine amax sweep
    (64, 14336, 0, 2, 4, False, "rms"),
    (5, 2048, 0, 3, 8, True, "rms"),        # OR-ed metadata fields
    (1, 256, 0, 2, 4, False, "layer"),
]


@pytest.mark.parametrize("m_tok,k,fmt,n,m,affine,norm", CASES)
def test_prepare_add_matches_oracle_and_unfused(sq, m_tok, k, fmt, n, m, affine, norm):
    h = synth.activations_student(500 + m_tok, m_tok, k)
    d = synth.activations_student(600 + m_tok, m_tok, k, outlier_frac=0.0)
    g = b = None
    if affine:
        g, b = synth.ln_params(9, k)
        if norm == "rms":
            b = None
    cg = None if g is None else cuda16(g)
    cb = None if b is None else cuda16(b)
    x_gpu, p = sq.prepare_add(cuda16(h), cuda16(d), cg, cb, 1e-5, n, m, fmt, norm=norm)
    x_oracle = oracle.add_fp16(h, d)
    assert_bits_equal("x = RN16(h + d)", x_gpu.cpu().numpy().view(np.uint16), x_oracle)
    ex = sq.prep_export(p)
    op = oracle.prepare(x_oracle, g, b, 1e-5, n, m, fmt, norm=norm)
    assert_prep_matches(ex, op)
    ref = sq.prep_export(sq.prepare(cuda16(x_oracle), cg, cb, 1e-5, n, m, fmt, norm=norm))
    for key in ["idx", "s_codes", "s_scales", "r_codes", "r_scales", "mu", "rstd"]:
        assert np.array_equal(np.asarray(ex[key]).view(np.uint8), np.asarray(ref[key]).view(np.uint8)), key
    assert sq.get_last_error() == sq.OK


def test_prepare_add_in_place(sq):
    h = synth.activations_student(700, 200, 4096)
    d = synth.activations_student(701, 200, 4096)
    ht = cuda16(h)
    x, p = sq.prepare_add(ht, cuda16(d), None, None, 1e-5, 2, 4, 0, x_out=ht)
    assert x.data_ptr() == ht.data_ptr()
    x_oracle = oracle.add_fp16(h, d)
    assert_bits_equal("x in place", ht.cpu().numpy().view(np.uint16), x_oracle)
    assert_prep_matches(sq.prep_export(p), oracle.prepare(x_oracle, None, None, 1e-5, 2, 4, 0))
    assert sq.get_last_error() == sq.OK


def test_prepare_add_rejects_partial_overlap(sq):
    h = torch.zeros((64, 512), dtype=torch.float16, device="cuda")
    d = torch.zeros((65, 512), dtype=torch.float16, device="cuda")
    with pytest.raises(sq.SharqError) as e:
        sq.prepare_add(h, d[:64], x_out=d[1:])
    assert e.value.status == sq.ERR_INVALID_ARG
