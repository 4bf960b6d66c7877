"""Argument checks of the Python binding: they raise ValueError before any
library call (and so also under python -O), so that no host pointer, wrong
dtype or strided tensor ever reaches a kernel. Runs without a GPU."""
import pytest
import torch

import sparsity_gemm_b200 as sq


def _cpu16(*shape):
    return torch.zeros(shape, dtype=torch.float16)


def test_prepare_rejects_host_and_mistyped_inputs():
    with pytest.raises(ValueError, match="CUDA tensor"):
        sq.prepare(_cpu16(16, 256))
    with pytest.raises(ValueError, match="fp16"):
        sq.prepare(torch.zeros((16, 256), dtype=torch.float32))
    with pytest.raises(ValueError, match="fp16"):
        sq.prepare(_cpu16(256, 32).t())  # strided
    with pytest.raises(ValueError, match="RMSNorm takes no ln_b"):
        sq.prepare(_cpu16(16, 256), None, _cpu16(256), norm="rms")
    with pytest.raises(ValueError, match='"layer" or "rms"'):
        sq.prepare(_cpu16(16, 256), norm="batch")


def test_weight_quantizers_reject_host_inputs():
    with pytest.raises(ValueError, match="CUDA tensor"):
        sq.quantize_weight(_cpu16(64, 256))
    with pytest.raises(ValueError, match="3 dimensions"):
        sq.quantize_weight_grouped(_cpu16(64, 256))
    with pytest.raises(ValueError, match="at least one"):
        sq.quantize_weight_fused([])
    with pytest.raises(ValueError, match="CUDA tensor"):
        sq.quantize_weight_fused([_cpu16(64, 256), _cpu16(32, 256)])


def test_linear_rejects_host_buffers():
    prep = sq.Prepared(torch.zeros(1024, dtype=torch.uint8), sq.SharqPrep())
    qw = sq.QuantizedWeight(torch.zeros(1024, dtype=torch.uint8), sq.SharqWQ())
    with pytest.raises(ValueError, match="prep.buf must be a CUDA tensor"):
        sq.linear(prep, qw)
    with pytest.raises(ValueError, match="prep.buf must be a CUDA tensor"):
        sq.linear(prep, qw, out=_cpu16(0, 0), bias=_cpu16(0))


def test_grouped_calls_reject_mistyped_offsets():
    prep = sq.Prepared(torch.zeros(1024, dtype=torch.uint8), sq.SharqPrep())
    with pytest.raises(ValueError, match="int32 vector"):
        sq.gather_rows(prep, None, torch.zeros(3, dtype=torch.int64), 0)
    with pytest.raises(ValueError, match="x must be a CUDA tensor"):
        sq.prepare_grouped(_cpu16(8, 256), torch.zeros(3, dtype=torch.int64))
    with pytest.raises(ValueError, match="offsets must be a CUDA tensor"):
        sq.gather_rows(prep, None, torch.zeros(3, dtype=torch.int32), 0)
    qw = sq.QuantizedWeight(torch.zeros(1024, dtype=torch.uint8), sq.SharqWQ())
    with pytest.raises(ValueError, match="int32 vector"):
        sq.linear_grouped(prep, torch.zeros(3, dtype=torch.float32), qw, 0)


def test_group_view_range():
    d = sq.SharqWQ()
    d.groups = 2
    qw = sq.QuantizedWeight(torch.zeros(16, dtype=torch.uint8), d)
    with pytest.raises(ValueError, match="out of range"):
        sq.group_view(qw, 2)


class _AsCuda(torch.Tensor):
    """A host tensor that reports itself as living on cuda:0, so that the
    binding's checks can be driven on a machine without a GPU."""

    @property
    def is_cuda(self):
        return True

    @property
    def device(self):
        return torch.device("cuda", 0)


def _as_cuda(t):
    return t.as_subclass(_AsCuda)


def test_valid_arguments_pass_the_checks_and_reach_the_library(monkeypatch):
    from unittest import mock
    fake = mock.MagicMock()
    for name in ("sharq_weight_bytes", "sharq_prep_bytes", "sharq_weight_bytes_grouped", "sharq_gather_bytes",
                 "sharq_weight_bytes_fused"):
        getattr(fake, name).return_value = 4096
    monkeypatch.setattr(sq, "lib", lambda: fake)
    monkeypatch.setattr(sq, "_device_buffer", lambda n, dev: _as_cuda(torch.zeros(max(n, 1), dtype=torch.uint8)))
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a: mock.Mock(cuda_stream=0))
    for name in ("sharq_quantize_weight", "sharq_prepare", "sharq_prepare_rms", "sharq_linear", "sharq_linear_bias",
                 "sharq_quantize_weight_fused", "sharq_quantize_weight_grouped", "sharq_gather_rows",
                 "sharq_prepare_grouped", "sharq_linear_grouped"):
        getattr(fake, name).return_value = sq.OK

    x = _as_cuda(_cpu16(16, 256))
    g = _as_cuda(_cpu16(256))
    p = sq.prepare(x, g, g)
    sq.prepare(x, g, None, norm="rms", out=p)
    qw = sq.quantize_weight(_as_cuda(_cpu16(64, 256)))
    p.desc.m_tok, qw.desc.n_out = 16, 64  # what the library would have filled in
    sq.linear(p, qw, out=_as_cuda(_cpu16(16, 64)), bias=_as_cuda(_cpu16(64)))
    sq.quantize_weight_fused([_as_cuda(_cpu16(64, 256)), _as_cuda(_cpu16(32, 256))])
    qg = sq.quantize_weight_grouped(_as_cuda(_cpu16(2, 64, 256)))
    off = _as_cuda(torch.zeros(3, dtype=torch.int32))
    gp = sq.gather_rows(p, _as_cuda(torch.zeros(4, dtype=torch.int32)), off, 4)
    sq.prepare_grouped(x, off, g, None, norm="rms", out=gp)
    qg.desc.n_out = 64
    sq.linear_grouped(gp, off, qg, 4, out=_as_cuda(_cpu16(4, 64)))
    for name in ("sharq_prepare", "sharq_prepare_rms", "sharq_quantize_weight", "sharq_linear_bias",
                 "sharq_quantize_weight_fused", "sharq_quantize_weight_grouped", "sharq_gather_rows",
                 "sharq_prepare_grouped", "sharq_linear_grouped"):
        assert getattr(fake, name).called, name
