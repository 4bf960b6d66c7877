"""sharq_prepare_noalloc: the preparation operator for callers that cannot
allocate device memory (a plugin handed only its input and output tensors, a
latency-critical path that must not call cudaMalloc, a deployment whose
device memory is planned ahead). Its working memory lives in a fixed array
inside the library, so the caller provides only inputs and outputs.

Checked here through the C ABI: on two calls in a row (different inputs,
so stale state in the shared array would show), its outputs equal the CPU
oracle's bit for bit (codes, scales, mask, statistics, tensor scale) and
those of sharq_prepare, and the dual-path linear on its outputs is within
the GEMM tolerance of the oracle's and equal to the linear on sharq_prepare's
outputs. The shapes reach every statistics path of sharq_prepare (the
single-launch cluster kernel for up to 8 rows, the warp-per-row kernel, and
its certified sums for rows longer than 2048 elements), so the equality
covers each of them against the one-CTA-per-row kernel used here. This file
is collected last and also passes on its own in a fresh process.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import assert_linear_close, assert_prep_matches

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


def _check_pair(sq, x, g, b, n, m, fmt, qw, w_oracle, call):
    m_tok, k = x.shape
    ref = sq.prepare(x, g, b, 1e-5, n, m, fmt)
    st, got, _ = _prepare_noalloc(sq, x, n, m, fmt, 1e-5, g, b)
    assert st == sq.OK, sq.status_name(st)
    assert sq.last_launch_count() == 2  # statistics and encode
    ea, eb = sq.prep_export(ref), sq.prep_export(got)
    for key in ["idx", "s_codes", "s_scales", "r_codes", "r_scales", "mu", "rstd"]:
        assert np.array_equal(np.asarray(ea[key]).view(np.uint8), np.asarray(eb[key]).view(np.uint8)), (call, key)
    assert np.float32(ea["s_t"]) == np.float32(eb["s_t"])
    # against the oracle itself, not only against the other entry point
    xh = x.cpu().numpy().view(np.uint16)
    gh = None if g is None else g.cpu().numpy().view(np.uint16)
    bh = None if b is None else b.cpu().numpy().view(np.uint16)
    op = oracle.prepare(xh, gh, bh, 1e-5, n, m, fmt)
    assert_prep_matches(eb, op)
    out_ref = sq.linear(ref, qw).cpu().numpy()
    out_got = sq.linear(got, qw).cpu().numpy()
    # same prepared bits and the same kernel: identical outputs
    assert np.array_equal(out_ref, out_got)
    rows = np.arange(min(m_tok, 24))
    want, bound = oracle.linear_prepared(op, w_oracle, rows=rows)
    assert_linear_close(out_got[rows], want, bound)
    assert sq.get_last_error() == sq.OK


# (fmt, n, m, affine, k, rows of the two calls): 300 / 129 rows reach the
# warp-per-row statistics, 1 / 8 rows the single-launch cluster kernel,
# k = 4096 and 14336 the certified sums
CASES = [(0, 2, 4, False, 1024, (300, 129)), (1, 4, 8, True, 1024, (300, 129)),
         (0, 2, 4, False, 4096, (1, 8)), (0, 2, 4, True, 4096, (8, 1)),
         (0, 2, 4, False, 14336, (40, 3))]


@pytest.mark.parametrize("fmt,n,m,affine,k,rows", CASES)
def test_noalloc_prepare_matches_oracle_and_prepare_on_consecutive_calls(sq, fmt, n, m, affine, k, rows):
    w_h = synth.weights(71, 288, k)
    qw = sq.quantize_weight(_cuda16(w_h), fmt)
    w_oracle = oracle.quantize_weight(w_h.view(np.uint16), fmt)
    g, b = (synth.ln_params(72, k) if affine else (None, None))
    g = None if g is None else _cuda16(g)
    b = None if b is None else _cuda16(b)
    for call, m_tok in enumerate(rows):  # two calls in a row
        x = _cuda16(synth.activations_student(73 + call, m_tok, k))
        _check_pair(sq, x, g, b, n, m, fmt, qw, w_oracle, call)


def test_noalloc_rejects_more_rows_than_its_array_holds(sq):
    k = 256
    limit = 16384  # SHARQ_NOALLOC_MAX_ROWS
    x = torch.zeros((limit + 1, k), dtype=torch.float16, device="cuda")
    st, _, _ = _prepare_noalloc(sq, x, 2, 4, 0)
    assert st == sq.ERR_UNSUPPORTED
    st, _, _ = _prepare_noalloc(sq, x[:limit], 2, 4, 0)
    assert st == sq.OK
    assert sq.get_last_error() == sq.OK
