"""The C ABI on the host (no GPU): the library loads, exports every entry
point include/sharq.h declares, its structs match the header byte for byte,
and host-side validation rejects bad arguments before touching CUDA."""
import ctypes as C
import os
import re
import subprocess

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "sharq.h")


@pytest.fixture(scope="module")
def sq():
    from sparsity_gemm_b200 import build
    build.build()
    import sparsity_gemm_b200 as sq
    sq.lib()
    return sq


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sharq_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared()
    for required in ["sharq_quantize_weight", "sharq_prepare", "sharq_linear", "sharq_prep_bytes",
                     "sharq_weight_bytes", "sharq_get_last_error"]:
        assert required in names


def test_library_exports_every_declared_symbol(sq):
    out = subprocess.run(["nm", "-D", "--defined-only", sq.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (sharq_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(sq.lib(), n)


def test_struct_layout_matches_header(sq, tmp_path):
    fields = {
        "sharq_wq": [f for f, _ in sq.SharqWQ._fields_],
        "sharq_prep": [f for f, _ in sq.SharqPrep._fields_],
    }
    src = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', "int main(void) {"]
    for st, fs in fields.items():
        src.append(f'printf("{st} %zu\\n", sizeof({st}));')
        for f in fs:
            src.append(f'printf("{st}.{f} %zu\\n", offsetof({st}, {f}));')
    src.append("return 0; }")
    c = tmp_path / "layout.c"
    c.write_text("\n".join(src))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", str(c), "-o", str(exe)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True).stdout.splitlines())
    for st, cls in [("sharq_wq", sq.SharqWQ), ("sharq_prep", sq.SharqPrep)]:
        assert int(got[st]) == C.sizeof(cls)
        for f, _ in cls._fields_:
            assert int(got[f"{st}.{f}"]) == getattr(cls, f).offset, (st, f)


def test_size_queries(sq):
    assert sq.weight_bytes(256, 256, sq.NVFP4) > 256 * 128
    assert sq.weight_bytes(256, 300, sq.NVFP4) == 0      # k not a multiple of 256
    assert sq.weight_bytes(250, 256, sq.NVFP4) == 0      # n_out not a multiple of 32
    assert sq.weight_bytes(256, 256, 5) == 0
    assert sq.prep_bytes(16, 256, 2, 4, sq.NVFP4) > 2 * 16 * 128
    assert sq.prep_bytes(0, 256, 2, 4, sq.NVFP4) > 0      # empty activations are valid
    assert sq.prep_bytes(16, 256, 5, 4, sq.NVFP4) == 0    # n > m
    assert sq.prep_bytes(16, 256, 2, 3, sq.NVFP4) == 0    # m not in {2,4,8,16}
    assert sq.prep_bytes(16, 65536 + 256, 2, 4, sq.NVFP4) == 0
    assert sq.prep_bytes(-1, 256, 2, 4, sq.MXFP4) == 0
    a = sq.prep_bytes(128, 4096, 2, 4, sq.NVFP4)
    b = sq.prep_bytes(256, 4096, 2, 4, sq.NVFP4)
    assert b > a
    # codes dominate: two [m_tok, k/2] code matrices plus scales and metadata
    assert b >= 2 * 256 * 2048 + 2 * 256 * 256 + 256 * 512


def test_prepare_rejects_bad_arguments_without_cuda(sq):
    L = sq.lib()
    fake = C.c_void_p(1 << 20)  # aligned, never dereferenced: validation fails first
    desc = sq.SharqPrep()
    big = 1 << 30

    def call(x=fake, m_tok=16, k=256, g=None, b=None, eps=1e-5, n=2, m=4, fmt=0, buf=fake, nbytes=big):
        return L.sharq_prepare(x, m_tok, k, g, b, eps, n, m, fmt, buf, nbytes, C.byref(desc), None)

    assert call(k=300) == sq.ERR_INVALID_ARG
    assert call(n=5) == sq.ERR_INVALID_ARG
    assert call(m=6, n=2) == sq.ERR_INVALID_ARG
    assert call(fmt=2) == sq.ERR_INVALID_ARG
    assert call(eps=0.0) == sq.ERR_INVALID_ARG
    assert call(eps=float("nan")) == sq.ERR_INVALID_ARG
    assert call(eps=-1e-5) == sq.ERR_INVALID_ARG
    assert call(buf=None) == sq.ERR_INVALID_ARG
    assert call(x=None) == sq.ERR_INVALID_ARG
    assert call(nbytes=10) == sq.ERR_INVALID_ARG
    assert call(x=C.c_void_p((1 << 20) + 8)) == sq.ERR_INVALID_ARG      # x not 16-byte aligned
    assert call(buf=C.c_void_p((1 << 20) + 128)) == sq.ERR_INVALID_ARG  # buffer not 256-byte aligned
    assert call(g=C.c_void_p((1 << 20) + 2)) == sq.ERR_INVALID_ARG


def test_quantize_weight_rejects_bad_arguments_without_cuda(sq):
    L = sq.lib()
    fake = C.c_void_p(1 << 20)
    desc = sq.SharqWQ()
    assert L.sharq_quantize_weight(fake, 250, 256, 0, fake, 1 << 30, C.byref(desc), None) == sq.ERR_INVALID_ARG
    assert L.sharq_quantize_weight(fake, 256, 256, 0, fake, 16, C.byref(desc), None) == sq.ERR_INVALID_ARG
    assert L.sharq_quantize_weight(None, 256, 256, 0, fake, 1 << 30, C.byref(desc), None) == sq.ERR_INVALID_ARG
    assert L.sharq_quantize_weight(fake, 256, 256, 3, fake, 1 << 30, C.byref(desc), None) == sq.ERR_INVALID_ARG


def test_linear_rejects_mismatched_handles_without_cuda(sq):
    L = sq.lib()
    p = sq.SharqPrep(m_tok=16, k=256, n=2, m=4, fmt=0, sf_rows=128, meta_row_bytes=32,
                     s_codes=1 << 20, r_codes=1 << 21)
    w = sq.SharqWQ(n_out=256, k=256, fmt=0, sf_rows=256, codes=1 << 22, scales_backbone=1 << 23,
                   scales_residual=1 << 23)
    out = C.c_void_p(1 << 24)
    w.fmt = 1
    assert L.sharq_linear(C.byref(p), C.byref(w), out, None) == sq.ERR_INVALID_ARG
    w.fmt = 0
    w.k = 512
    assert L.sharq_linear(C.byref(p), C.byref(w), out, None) == sq.ERR_INVALID_ARG
    w.k = 256
    assert L.sharq_linear(C.byref(p), C.byref(w), None, None) == sq.ERR_INVALID_ARG
    w.scales_residual = 1 << 25  # the two scale views must hold the same values
    assert L.sharq_linear(C.byref(p), C.byref(w), out, None) == sq.ERR_INVALID_ARG
    w.scales_residual = 1 << 23
    # the epilogue writes whole 32-byte sectors: a 16-byte aligned output is refused
    assert L.sharq_linear(C.byref(p), C.byref(w), C.c_void_p((1 << 24) + 16), None) == sq.ERR_INVALID_ARG
    w.groups = 3  # stacked weights go to sharq_linear_grouped
    assert L.sharq_linear(C.byref(p), C.byref(w), out, None) == sq.ERR_INVALID_ARG
    w.groups = 1
    assert L.sharq_linear(None, C.byref(w), out, None) == sq.ERR_INVALID_ARG
    p.m_tok = 0  # empty activations: nothing to do
    assert L.sharq_linear(C.byref(p), C.byref(w), None, None) == sq.OK


def test_fused_weights_and_bias_validation_without_cuda(sq):
    L = sq.lib()
    rows = lambda *r: (C.c_int64 * len(r))(*r)
    assert L.sharq_weight_bytes_fused(rows(4096, 1024, 1024), 3, 4096, 0) == sq.weight_bytes(6144, 4096, 0)
    assert L.sharq_weight_bytes_fused(rows(64, 48), 2, 256, 0) == 0          # 48 is not a multiple of 32
    assert L.sharq_weight_bytes_fused(rows(64, 0), 2, 256, 0) == 0
    assert L.sharq_weight_bytes_fused(rows(*([32] * 9)), 9, 256, 0) == 0     # more than SHARQ_SEGMENTS_MAX
    assert L.sharq_weight_bytes_fused(None, 1, 256, 0) == 0
    desc = sq.SharqWQ()
    assert L.sharq_quantize_weight_fused(C.c_void_p(1 << 20), rows(64, 48), 2, 256, 0, C.c_void_p(1 << 21),
                                         1 << 20, C.byref(desc), None) == sq.ERR_INVALID_ARG
    p = sq.SharqPrep(m_tok=16, k=256, n=2, m=4, fmt=0, sf_rows=128, meta_row_bytes=32,
                     s_codes=1 << 20, r_codes=1 << 21)
    w = sq.SharqWQ(n_out=256, k=256, fmt=0, sf_rows=256, codes=1 << 22, scales_backbone=1 << 23,
                   scales_residual=1 << 23)
    out = C.c_void_p(1 << 24)
    w.segments = 2
    w.seg_end[0], w.seg_end[1] = 128, 200   # the last segment must end at n_out
    assert L.sharq_linear(C.byref(p), C.byref(w), out, None) == sq.ERR_INVALID_ARG
    w.seg_end[0], w.seg_end[1] = 100, 256   # boundaries are multiples of 32
    assert L.sharq_linear(C.byref(p), C.byref(w), out, None) == sq.ERR_INVALID_ARG
    w.seg_end[0], w.seg_end[1] = 256, 256   # strictly increasing
    assert L.sharq_linear(C.byref(p), C.byref(w), out, None) == sq.ERR_INVALID_ARG
    w.segments = 9
    assert L.sharq_linear(C.byref(p), C.byref(w), out, None) == sq.ERR_INVALID_ARG
    w.segments = 1
    # the bias must be 16-byte aligned
    assert L.sharq_linear_bias(C.byref(p), C.byref(w), C.c_void_p((1 << 25) + 8), out, None) == sq.ERR_INVALID_ARG
    w.segments, w.groups = 2, 2
    w.seg_end[0], w.seg_end[1] = 128, 256   # stacked experts cannot also be fused
    assert L.sharq_linear_grouped(C.byref(p), C.c_void_p(1 << 26), 2, 16, C.byref(w), out,
                                  None) == sq.ERR_INVALID_ARG


def test_status_strings(sq):
    assert sq.status_name(0) == "SHARQ_OK"
    assert sq.status_name(4) == "SHARQ_ERR_TIMEOUT"
