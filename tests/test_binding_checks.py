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
