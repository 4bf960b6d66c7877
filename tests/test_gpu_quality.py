"""Quality check of the dual-path linear (reported by bench.py, checked here
as a property): on outlier-heavy activations, the SharQ output is closer
than plain NVFP4 (the same library with n = m and the residual codes
zeroed) both to an fp16 GEMM of RN16(LayerNorm(x)) W^T and, isolating the
activation side, to RN16(LayerNorm(x)) deq(Q(W))^T: the point of the
residual path. Both outputs share Q(W), whose error dominates against the
fp16 weight."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sq():
    import sparsity_gemm_b200 as sq
    assert torch.cuda.is_available()
    sq.lib()
    return sq


E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def _deq_weight(sq, qw):
    wx = sq.weight_export(qw)
    sc = torch.from_numpy(wx["scales"]).cuda()
    sv = sc.view(torch.float8_e4m3fn).float() if qw.desc.fmt == sq.NVFP4 else torch.exp2(sc.float() - 127.0)
    vals = torch.tensor(E2M1, device="cuda")[torch.from_numpy(wx["codes"]).cuda().long()]
    return vals * sv.repeat_interleave(sq.BLOCK[qw.desc.fmt], dim=1) * float(wx["s_tw"])


def _cuda16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.float16)).cuda()


@pytest.mark.parametrize("fmt,n,m", [(0, 2, 4), (1, 2, 4), (0, 4, 8)])
def test_sharq_error_below_plain_fp4(sq, fmt, n, m):
    rows, k, n_out = 512, 2048, 768
    x = _cuda16(synth.activations_student(400 + fmt, rows, k))
    w = _cuda16(synth.weights(401, n_out, k))
    x_ln = torch.nn.functional.layer_norm(x.float(), (k,), eps=1e-5).half().float()
    qw = sq.quantize_weight(w, fmt)
    out = sq.linear(sq.prepare(x, None, None, 1e-5, n, m, fmt), qw).float()
    plain = sq.prepare(x, None, None, 1e-5, m, m, fmt)
    off = plain.desc.r_codes - plain.buf.data_ptr()
    plain.buf[off:off + rows * k // 2].zero_()
    out_plain = sq.linear(plain, qw).float()
    assert sq.get_last_error() == sq.OK
    errs = {}
    for tag, wref in (("fp16 W", w.float()), ("deq Q(W)", _deq_weight(sq, qw))):
        ref = x_ln @ wref.t()
        nref = torch.linalg.vector_norm(ref).item()
        errs[tag] = (torch.linalg.vector_norm(out - ref).item() / nref,
                     torch.linalg.vector_norm(out_plain - ref).item() / nref)
    print(errs)
    e_sharq, e_plain = errs["fp16 W"]
    assert 0.01 < e_plain < 0.5, e_plain
    for tag, (e_sharq, e_plain) in errs.items():
        assert e_sharq < e_plain, (tag, e_sharq, e_plain)
