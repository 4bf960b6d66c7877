"""sharq_prepare_noalloc: the preparation operator for callers that cannot
allocate device memory (a plugin handed only its input and output tensors, a
latency-critical path that must not call cudaMalloc, a deployment whose
device memory is planned ahead). Its working memory lives in a fixed array
inside the library, so the caller provides only inputs and outputs.

Checked here through the C ABI: on two calls in a row (different inputs,
so stale state in the shared array would show), its outputs equal those of
sharq_prepare bit for bit, and the dual-path linear on its outputs equals
the linear on sharq_prepare's outputs. This file is collected last and also
passes on its own in a fresh process.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _buf(nbytes):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device="cuda")


def _prepare_noalloc(sq, x, n, m, fmt, eps=1e-5, ln_w=None, ln_b=None):
    """Calls the entry point through the C ABI with caller-allocated outputs
    sized by the layouts the header documents."""
    m_tok, k = x.shape
    blk = sq.BLOCK[fmt]
    sf_rows = max(128, (m_tok + 127) // 128 * 128)
    ib = 1 if m <= 2 else 2 if m <= 4 else 3 if m <= 8 else 4
    meta_row = ((k // m) * n * ib + 7) // 8
    outs = dict(s_codes=_buf(m_tok * k // 2), r_codes=_buf(m_tok * k // 2),
                s_scales=_buf(sf_rows * k // blk), r_scales=_buf(sf_rows * k // blk),
                meta=_buf(m_tok * meta_row), s_t=torch.empty(64, dtype=torch.float32, device="cuda"))
    desc = sq.SharqPrep()
    p = lambda t: None if t is None else C.c_void_p(t.data_ptr())
    st = sq.lib().sharq_prepare_noalloc(
        p(x), m_tok, k, p(ln_w), p(ln_b), C.c_float(eps), n, m, fmt,
        p(outs["s_codes"]), p(outs["r_codes"]), p(outs["s_scales"]), p(outs["r_scales"]),
        p(outs["meta"]), p(outs["s_t"]), C.byref(desc), C.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, sq.Prepared(outs["s_codes"], desc), outs


@pytest.fixture(scope="module")
def sq():
    import sparsity_gemm_b200 as sq
    assert torch.cuda.is_available()
    L = sq.lib()
    L.sharq_prepare_noalloc.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p, C.c_float,
                                        C.c_int, C.c_int, C.c_int] + [C.c_void_p] * 6 + \
                                       [C.POINTER(sq.SharqPrep), C.c_void_p]
    L.sharq_prepare_noalloc.restype = C.c_int
    return sq


def _cuda16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.float16)).cuda()


@pytest.mark.parametrize("fmt,n,m,affine", [(0, 2, 4, False), (1, 4, 8, True)])
def test_noalloc_prepare_matches_prepare_on_consecutive_calls(sq, fmt, n, m, affine):
    k = 1024
    w = _cuda16(synth.weights(71, 544, k))
    qw = sq.quantize_weight(w, fmt)
    g, b = (synth.ln_params(72, k) if affine else (None, None))
    g = None if g is None else _cuda16(g)
    b = None if b is None else _cuda16(b)
    for call, (seed, m_tok) in enumerate([(73, 300), (74, 129)]):  # two calls in a row
        x = _cuda16(synth.activations_student(seed, m_tok, k))
        ref = sq.prepare(x, g, b, 1e-5, n, m, fmt)
        st, got, _ = _prepare_noalloc(sq, x, n, m, fmt, 1e-5, g, b)
        assert st == sq.OK, sq.status_name(st)
        ea, eb = sq.prep_export(ref), sq.prep_export(got)
        for key in ["idx", "s_codes", "s_scales", "r_codes", "r_scales", "mu", "rstd"]:
            assert np.array_equal(np.asarray(ea[key]).view(np.uint8), np.asarray(eb[key]).view(np.uint8)), (call, key)
        assert np.float32(ea["s_t"]) == np.float32(eb["s_t"])
        out_ref = sq.linear(ref, qw).cpu().numpy().astype(np.float64)
        out_got = sq.linear(got, qw).cpu().numpy().astype(np.float64)
        # same prepared bits and the same kernel: identical outputs, which is
        # within the tolerance every GEMM test uses (1e-3 sum|a||w|)
        assert np.array_equal(out_ref, out_got)
        assert sq.get_last_error() == sq.OK


def test_noalloc_rejects_more_rows_than_its_array_holds(sq):
    k = 256
    limit = 16384  # SHARQ_NOALLOC_MAX_ROWS
    x = torch.zeros((limit + 1, k), dtype=torch.float16, device="cuda")
    st, _, _ = _prepare_noalloc(sq, x, 2, 4, 0)
    assert st == sq.ERR_UNSUPPORTED
    st, _, _ = _prepare_noalloc(sq, x[:limit], 2, 4, 0)
    assert st == sq.OK
    assert sq.get_last_error() == sq.OK
