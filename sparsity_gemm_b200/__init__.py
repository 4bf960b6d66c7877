"""SharQ per-linear-layer hot path on NVIDIA B200 (sm_100a).

A thin binding over the C ABI of libsharq.so (include/sharq.h): it allocates
caller-owned buffers with torch, passes raw device pointers and the current
CUDA stream, and checks status codes. Every step of the path runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback, and importing
the package fails loudly when the library is missing.

Method: "SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM
Inference" (arXiv 2606.26587), Abstract.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsharq.so")

NVFP4, MXFP4 = 0, 1
BLOCK = {NVFP4: 16, MXFP4: 32}
K_ALIGN, K_MAX, N_ALIGN = 256, 65536, 32
SEGMENTS_MAX = 8

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = 0, 1, 2, 3, 4


class SharqError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_name(status)}")
        self.status = status


class SharqWQ(C.Structure):
    _fields_ = [("n_out", C.c_int64), ("k", C.c_int64), ("fmt", C.c_int32), ("groups", C.c_int32),
                ("sf_rows", C.c_int64), ("codes", C.c_void_p), ("scales_backbone", C.c_void_p),
                ("scales_residual", C.c_void_p), ("tensor_scale", C.c_void_p), ("scratch", C.c_void_p),
                ("segments", C.c_int32), ("seg_end", C.c_int32 * SEGMENTS_MAX), ("sparse", C.c_int32)]


class SharqPrep(C.Structure):
    _fields_ = [("m_tok", C.c_int64), ("k", C.c_int64), ("n", C.c_int32), ("m", C.c_int32),
                ("fmt", C.c_int32), ("groups", C.c_int32), ("sf_rows", C.c_int64),
                ("meta_row_bytes", C.c_int64), ("s_codes", C.c_void_p), ("r_codes", C.c_void_p),
                ("s_scales", C.c_void_p), ("r_scales", C.c_void_p), ("meta", C.c_void_p),
                ("tensor_scale", C.c_void_p), ("scratch", C.c_void_p), ("sparse", C.c_int32)]


_lib = None


def lib():
    """The loaded libsharq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sparsity_gemm_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i64, i32, f32, sz = C.c_void_p, C.c_int64, C.c_int, C.c_float, C.c_size_t
        L.sharq_weight_bytes.argtypes = [i64, i64, i32]
        L.sharq_weight_bytes.restype = sz
        L.sharq_prep_bytes.argtypes = [i64, i64, i32, i32, i32]
        L.sharq_prep_bytes.restype = sz
        L.sharq_quantize_weight.argtypes = [vp, i64, i64, i32, vp, sz, C.POINTER(SharqWQ), vp]
        L.sharq_prepare.argtypes = [vp, i64, i64, vp, vp, f32, i32, i32, i32, vp, sz, C.POINTER(SharqPrep), vp]
        L.sharq_prepare_rms.argtypes = [vp, i64, i64, vp, f32, i32, i32, i32, vp, sz, C.POINTER(SharqPrep), vp]
        L.sharq_linear.argtypes = [C.POINTER(SharqPrep), C.POINTER(SharqWQ), vp, vp]
        L.sharq_prep_export.argtypes = [C.POINTER(SharqPrep)] + [vp] * 8 + [vp]
        L.sharq_weight_export.argtypes = [C.POINTER(SharqWQ), vp, vp, vp, vp, vp]
        L.sharq_get_last_error.argtypes = [vp]
        L.sharq_last_timeout_site.restype = C.c_uint32
        L.sharq_set_wait_limit_ns.argtypes = [C.c_uint64]
        L.sharq_set_wait_limit_ns.restype = C.c_uint64
        L.sharq_selftest_wait.argtypes = [C.c_uint64, vp]
        L.sharq_selftest_wait.restype = i32
        L.sharq_selftest_division.argtypes = [C.c_uint64, C.c_uint64, C.POINTER(C.c_uint64), vp, vp]
        L.sharq_selftest_division.restype = i32
        L.sharq_weight_bytes_grouped.argtypes = [i64, i64, i64, i32]
        L.sharq_weight_bytes_grouped.restype = sz
        L.sharq_quantize_weight_grouped.argtypes = [vp, i64, i64, i64, i32, vp, sz, C.POINTER(SharqWQ), vp]
        L.sharq_grouped_rows.argtypes = [i64, i64]
        L.sharq_grouped_rows.restype = i64
        L.sharq_gather_bytes.argtypes = [i64, i64, i64, i32, i32, i32]
        L.sharq_gather_bytes.restype = sz
        L.sharq_gather_rows.argtypes = [C.POINTER(SharqPrep), vp, vp, i64, i64, vp, sz, C.POINTER(SharqPrep), vp]
        L.sharq_linear_grouped.argtypes = [C.POINTER(SharqPrep), vp, i64, i64, C.POINTER(SharqWQ), vp, vp]
        L.sharq_weight_bytes_fused.argtypes = [C.POINTER(C.c_int64), i32, i64, i32]
        L.sharq_weight_bytes_fused.restype = sz
        L.sharq_quantize_weight_fused.argtypes = [vp, C.POINTER(C.c_int64), i32, i64, i32, vp, sz,
                                                  C.POINTER(SharqWQ), vp]
        L.sharq_linear_bias.argtypes = [C.POINTER(SharqPrep), C.POINTER(SharqWQ), vp, vp, vp]
        L.sharq_weight_tensor_scales.argtypes = [C.POINTER(SharqWQ), vp, vp]
        L.sharq_prepare_grouped.argtypes = [vp, i64, i64, vp, i64, vp, vp, f32, i32, i32, i32, i32, vp, sz,
                                            C.POINTER(SharqPrep), vp]
        L.sharq_prepare_add.argtypes = [vp, vp, vp, i64, i64, vp, vp, f32, i32, i32, i32, i32, vp, sz,
                                        C.POINTER(SharqPrep), vp]
        L.sharq_prep_bytes_sparse.argtypes = [i64, i64, i32]
        L.sharq_prep_bytes_sparse.restype = sz
        L.sharq_prepare_sparse.argtypes = [vp, i64, i64, vp, vp, f32, i32, i32, vp, sz, C.POINTER(SharqPrep), vp]
        L.sharq_weight_bytes_sparse.argtypes = [i64, i64, i32]
        L.sharq_weight_bytes_sparse.restype = sz
        L.sharq_quantize_weight_sparse.argtypes = [vp, i64, i64, i32, vp, sz, C.POINTER(SharqWQ), vp]
        L.sharq_status_string.argtypes = [i32]
        L.sharq_status_string.restype = C.c_char_p
        L.sharq_last_launch_count.restype = i32
        for name in ("sharq_quantize_weight", "sharq_prepare", "sharq_linear", "sharq_prep_export",
                     "sharq_weight_export", "sharq_get_last_error", "sharq_quantize_weight_grouped",
                     "sharq_gather_rows", "sharq_linear_grouped", "sharq_prepare_rms",
                     "sharq_quantize_weight_fused", "sharq_linear_bias", "sharq_weight_tensor_scales",
                     "sharq_prepare_grouped", "sharq_prepare_sparse", "sharq_quantize_weight_sparse", "sharq_prepare_add"):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def status_name(status: int) -> str:
    return lib().sharq_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise SharqError(status, what)


def _stream(stream) -> C.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _require(cond: bool, what: str):
    """Argument check that survives python -O (raises ValueError)."""
    if not cond:
        raise ValueError(what)


def _cuda_here(t: torch.Tensor, name: str):
    """t must live on the current CUDA device: the library launches on the
    current device, and a host or other-device pointer would reach a kernel."""
    _require(isinstance(t, torch.Tensor) and t.is_cuda, f"{name} must be a CUDA tensor")
    cur = torch.cuda.current_device()
    _require(t.device.index == cur,
             f"{name} is on {t.device} but the current device is cuda:{cur} (call torch.cuda.set_device first)")


def _fp16_matrix(t: torch.Tensor, name: str, dims: int = 2):
    _require(isinstance(t, torch.Tensor) and t.dtype == torch.float16 and t.dim() == dims and t.is_contiguous(),
             f"{name} must be a contiguous fp16 tensor with {dims} dimensions")
    _cuda_here(t, name)


def _int32_vector(t: torch.Tensor, name: str):
    _require(isinstance(t, torch.Tensor) and t.dtype == torch.int32 and t.dim() == 1 and t.is_contiguous(),
             f"{name} must be a contiguous int32 vector")
    _cuda_here(t, name)


def weight_bytes(n_out: int, k: int, fmt: int) -> int:
    return int(lib().sharq_weight_bytes(n_out, k, fmt))


def prep_bytes(m_tok: int, k: int, n: int, m: int, fmt: int) -> int:
    return int(lib().sharq_prep_bytes(m_tok, k, n, m, fmt))


class QuantizedWeight:
    """One FP4 weight payload (codes + MMA scale view + tensor scale)."""

    def __init__(self, buf: torch.Tensor, desc: SharqWQ):
        self.buf, self.desc = buf, desc

    @property
    def n_out(self):
        return self.desc.n_out

    @property
    def k(self):
        return self.desc.k


class Prepared:
    """Outputs of the preparation operator for one activation tensor."""

    def __init__(self, buf: torch.Tensor, desc: SharqPrep):
        self.buf, self.desc = buf, desc

    @property
    def m_tok(self):
        return self.desc.m_tok


def _device_buffer(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def quantize_weight(w: torch.Tensor, fmt: int = NVFP4, stream=None) -> QuantizedWeight:
    """Offline FP4 quantization of W [n_out, k] (fp16, CUDA)."""
    _fp16_matrix(w, "w")
    n_out, k = w.shape
    nbytes = weight_bytes(n_out, k, fmt)
    if nbytes == 0:
        raise SharqError(ERR_INVALID_ARG, f"weight shape {tuple(w.shape)} fmt {fmt}")
    buf = _device_buffer(nbytes, w.device)
    desc = SharqWQ()
    _check(lib().sharq_quantize_weight(_ptr(w), n_out, k, fmt, _ptr(buf), nbytes, C.byref(desc), _stream(stream)),
           "sharq_quantize_weight")
    return QuantizedWeight(buf, desc)


def prepare(x: torch.Tensor, ln_w=None, ln_b=None, eps: float = 1e-5, n: int = 2, m: int = 4,
            fmt: int = NVFP4, out: Prepared | None = None, stream=None, norm: str = "layer") -> Prepared:
    """Fused preparation operator on x [m_tok, k] (fp16, CUDA). norm:
    "layer" (LayerNorm with ln_w, ln_b) or "rms" (RMSNorm with weight ln_w;
    ln_b must be None)."""
    _require(norm in ("layer", "rms") and (norm == "layer" or ln_b is None),
             'norm must be "layer" or "rms" (RMSNorm takes no ln_b)')
    _fp16_matrix(x, "x")
    for t, name in ((ln_w, "ln_w"), (ln_b, "ln_b")):
        if t is not None:
            _fp16_matrix(t.view(-1) if t.is_contiguous() else t, name, 1)
            _require(t.numel() == x.shape[1], f"{name} must have {x.shape[1]} elements")
    m_tok, k = x.shape
    nbytes = prep_bytes(m_tok, k, n, m, fmt)
    if nbytes == 0:
        raise SharqError(ERR_INVALID_ARG, f"prep shape {tuple(x.shape)} {n}:{m} fmt {fmt}")
    if out is None or out.buf.numel() < nbytes:
        buf = _device_buffer(nbytes, x.device)
    else:
        buf = out.buf
        _cuda_here(buf, "out.buf")
    desc = SharqPrep()
    xp = _ptr(x) if m_tok > 0 else None
    if norm == "rms":
        _check(lib().sharq_prepare_rms(xp, m_tok, k, _ptr(ln_w), float(eps), n, m, fmt, _ptr(buf), buf.numel(),
                                       C.byref(desc), _stream(stream)), "sharq_prepare_rms")
    else:
        _check(lib().sharq_prepare(xp, m_tok, k, _ptr(ln_w), _ptr(ln_b), float(eps), n, m, fmt, _ptr(buf),
                                   buf.numel(), C.byref(desc), _stream(stream)), "sharq_prepare")
    return Prepared(buf, desc)


def linear(prep: Prepared, qw: QuantizedWeight, out: torch.Tensor | None = None, stream=None,
           bias: torch.Tensor | None = None) -> torch.Tensor:
    """Dual-path FP4 linear: fp16 [m_tok, n_out] = (Q(S) + Q(R)) Q(W)^T, scaled,
    plus an optional fp16 bias [n_out]. A fused weight (quantize_weight_fused)
    gives its segments' outputs side by side."""
    _cuda_here(prep.buf, "prep.buf")
    _cuda_here(qw.buf, "qw.buf")
    if out is None:
        out = torch.empty((prep.m_tok, qw.n_out), dtype=torch.float16, device=prep.buf.device)
    _require(out.dtype == torch.float16 and out.is_contiguous() and tuple(out.shape) == (prep.m_tok, qw.n_out),
             f"out must be a contiguous fp16 tensor of shape {(prep.m_tok, qw.n_out)}")
    _cuda_here(out, "out")
    optr = _ptr(out) if out.numel() else None
    if bias is None:
        _check(lib().sharq_linear(C.byref(prep.desc), C.byref(qw.desc), optr, _stream(stream)), "sharq_linear")
    else:
        _require(bias.dtype == torch.float16 and bias.is_contiguous() and bias.numel() == qw.n_out,
                 f"bias must be a contiguous fp16 tensor of {qw.n_out} elements")
        _cuda_here(bias, "bias")
        _check(lib().sharq_linear_bias(C.byref(prep.desc), C.byref(qw.desc), _ptr(bias), optr, _stream(stream)),
               "sharq_linear_bias")
    return out


def quantize_weight_fused(ws, fmt: int = NVFP4, stream=None) -> QuantizedWeight:
    """Offline FP4 quantization of several weights that read the same input
    (q/k/v, gate/up), stacked along n_out into one payload; each keeps its own
    tensor scale, so the fused linear's columns equal the separate linears'.
    ws: list of fp16 CUDA tensors [n_g, k]."""
    ws = list(ws)
    _require(len(ws) > 0, "ws must hold at least one weight")
    for i, w in enumerate(ws):
        _require(isinstance(w, torch.Tensor) and w.dtype == torch.float16 and w.dim() == 2,
                 f"ws[{i}] must be an fp16 matrix")
        _cuda_here(w, f"ws[{i}]")
    k = ws[0].shape[1]
    _require(all(w.shape[1] == k for w in ws), "every weight of a fused payload must have the same k")
    rows = (C.c_int64 * len(ws))(*[w.shape[0] for w in ws])
    nbytes = int(lib().sharq_weight_bytes_fused(rows, len(ws), k, fmt))
    if nbytes == 0:
        raise SharqError(ERR_INVALID_ARG, f"fused weight segments {[tuple(w.shape) for w in ws]} fmt {fmt}")
    w = torch.cat([t.contiguous() for t in ws], 0)
    buf = _device_buffer(nbytes, w.device)
    desc = SharqWQ()
    _check(lib().sharq_quantize_weight_fused(_ptr(w), rows, len(ws), k, fmt, _ptr(buf), nbytes, C.byref(desc),
                                             _stream(stream)), "sharq_quantize_weight_fused")
    qw = QuantizedWeight(buf, desc)
    qw._src = w  # the stacked copy stays alive until the quantizer has read it
    return qw


def weight_tensor_scales(qw: QuantizedWeight, stream=None) -> np.ndarray:
    """The tensor scale s_tW of each segment of a weight (one for a plain weight)."""
    segs = max(1, qw.desc.segments)
    out = np.zeros(segs, np.float32)
    _check(lib().sharq_weight_tensor_scales(C.byref(qw.desc), out.ctypes.data_as(C.c_void_p), _stream(stream)),
           "sharq_weight_tensor_scales")
    return out


def prepare_add(h: torch.Tensor, d: torch.Tensor, ln_w=None, ln_b=None, eps: float = 1e-5, n: int = 2, m: int = 4,
                fmt: int = NVFP4, x_out: torch.Tensor | None = None, out: Prepared | None = None, stream=None,
                norm: str = "layer"):
    """Residual add fused with the preparation: x = RN16(h + d) (fp16 [m_tok,
    k], CUDA) is written to x_out (a new tensor if None; may be h itself) and
    prepared as prepare(x) would, with x's statistics taken in the add's pass.
    Returns (x_out, Prepared)."""
    _require(norm in ("layer", "rms") and (norm == "layer" or ln_b is None),
             'norm must be "layer" or "rms" (RMSNorm takes no ln_b)')
    _fp16_matrix(h, "h")
    _fp16_matrix(d, "d")
    _require(h.shape == d.shape, "h and d must have the same shape")
    if x_out is None:
        x_out = torch.empty_like(h)
    _fp16_matrix(x_out, "x_out")
    _require(x_out.shape == h.shape, "x_out must have the shape of h")
    for t, name in ((ln_w, "ln_w"), (ln_b, "ln_b")):
        if t is not None:
            _fp16_matrix(t.view(-1) if t.is_contiguous() else t, name, 1)
            _require(t.numel() == h.shape[1], f"{name} must have {h.shape[1]} elements")
    m_tok, k = h.shape
    nbytes = prep_bytes(m_tok, k, n, m, fmt)
    if nbytes == 0:
        raise SharqError(ERR_INVALID_ARG, f"prep shape {tuple(h.shape)} {n}:{m} fmt {fmt}")
    if out is None or out.buf.numel() < nbytes:
        buf = _device_buffer(nbytes, h.device)
    else:
        buf = out.buf
        _cuda_here(buf, "out.buf")
    desc = SharqPrep()
    p = (lambda t: _ptr(t) if m_tok > 0 else None)
    _check(lib().sharq_prepare_add(p(h), p(d), p(x_out), m_tok, k, _ptr(ln_w), _ptr(ln_b), float(eps),
                                   1 if norm == "rms" else 0, n, m, fmt, _ptr(buf), buf.numel(), C.byref(desc),
                                   _stream(stream)), "sharq_prepare_add")
    return x_out, Prepared(buf, desc)


def prepare_sparse(x: torch.Tensor, ln_w=None, ln_b=None, eps: float = 1e-5, fmt: int = NVFP4,
                   out: Prepared | None = None, stream=None, norm: str = "layer") -> Prepared:
    """The preparation operator in the pair-wise 4:8 mode (the pattern of the
    structured-sparse FP4 tensor-core MMA): x [m_tok, k] (fp16, CUDA); the
    backbone is stored K-compacted and feeds tcgen05.mma.sp in linear(), with
    a weight from quantize_weight_sparse."""
    _require(norm in ("layer", "rms") and (norm == "layer" or ln_b is None),
             'norm must be "layer" or "rms" (RMSNorm takes no ln_b)')
    _fp16_matrix(x, "x")
    for t, name in ((ln_w, "ln_w"), (ln_b, "ln_b")):
        if t is not None:
            _fp16_matrix(t.view(-1) if t.is_contiguous() else t, name, 1)
            _require(t.numel() == x.shape[1], f"{name} must have {x.shape[1]} elements")
    m_tok, k = x.shape
    nbytes = int(lib().sharq_prep_bytes_sparse(m_tok, k, fmt))
    if nbytes == 0:
        raise SharqError(ERR_INVALID_ARG, f"sparse prep shape {tuple(x.shape)} fmt {fmt}")
    if out is None or out.buf.numel() < nbytes:
        buf = _device_buffer(nbytes, x.device)
    else:
        buf = out.buf
        _cuda_here(buf, "out.buf")
    desc = SharqPrep()
    _check(lib().sharq_prepare_sparse(_ptr(x) if m_tok > 0 else None, m_tok, k, _ptr(ln_w), _ptr(ln_b), float(eps),
                                      1 if norm == "rms" else 0, fmt, _ptr(buf), buf.numel(), C.byref(desc),
                                      _stream(stream)), "sharq_prepare_sparse")
    return Prepared(buf, desc)


def quantize_weight_sparse(w: torch.Tensor, fmt: int = NVFP4, stream=None) -> QuantizedWeight:
    """Offline FP4 quantization of W [n_out, k] (fp16, CUDA) for the pair-wise
    4:8 mode: one scale per 32 (NVFP4) or 64 (MXFP4) values, which the
    backbone path reads as is and the residual path once per half block."""
    _fp16_matrix(w, "w")
    n_out, k = w.shape
    nbytes = int(lib().sharq_weight_bytes_sparse(n_out, k, fmt))
    if nbytes == 0:
        raise SharqError(ERR_INVALID_ARG, f"sparse weight shape {tuple(w.shape)} fmt {fmt}")
    buf = _device_buffer(nbytes, w.device)
    desc = SharqWQ()
    _check(lib().sharq_quantize_weight_sparse(_ptr(w), n_out, k, fmt, _ptr(buf), nbytes, C.byref(desc),
                                              _stream(stream)), "sharq_quantize_weight_sparse")
    return QuantizedWeight(buf, desc)


def prep_export(prep: Prepared, stream=None) -> dict:
    """Canonical host copies (numpy) of a prepared activation (pair-wise mode:
    backbone codes decompressed, one backbone scale per 2 blocks)."""
    d = prep.desc
    m_tok, k, blk = d.m_tok, d.k, BLOCK[d.fmt]
    sblk = 2 * blk if d.sparse else blk
    out = dict(
        idx=np.zeros((m_tok, k // d.m, d.n), np.uint8),
        s_codes=np.zeros((m_tok, k), np.uint8), s_scales=np.zeros((m_tok, k // sblk), np.uint8),
        r_codes=np.zeros((m_tok, k), np.uint8), r_scales=np.zeros((m_tok, k // blk), np.uint8),
        mu=np.zeros(m_tok, np.float32), rstd=np.zeros(m_tok, np.float32), s_t=np.zeros(1, np.float32))
    p = lambda a: a.ctypes.data_as(C.c_void_p)
    _check(lib().sharq_prep_export(C.byref(d), p(out["idx"]), p(out["s_codes"]), p(out["s_scales"]),
                                   p(out["r_codes"]), p(out["r_scales"]), p(out["mu"]), p(out["rstd"]),
                                   p(out["s_t"]), _stream(stream)), "sharq_prep_export")
    out["s_t"] = out["s_t"][0]
    return out


def weight_export(qw: QuantizedWeight, stream=None) -> dict:
    d = qw.desc
    blk = BLOCK[d.fmt]
    sblk = 2 * blk if d.sparse else blk
    out = dict(codes=np.zeros((d.n_out, d.k), np.uint8), scales=np.zeros((d.n_out, d.k // sblk), np.uint8),
               scales_residual=np.zeros((d.n_out, d.k // blk), np.uint8), s_tw=np.zeros(1, np.float32))
    p = lambda a: a.ctypes.data_as(C.c_void_p)
    _check(lib().sharq_weight_export(C.byref(d), p(out["codes"]), p(out["scales"]), p(out["scales_residual"]),
                                     p(out["s_tw"]), _stream(stream)), "sharq_weight_export")
    out["s_tw"] = out["s_tw"][0]
    return out


# ---------------------------------------------------------------------------
# Mixture-of-experts grouped variant


def quantize_weight_grouped(w: torch.Tensor, fmt: int = NVFP4, stream=None) -> QuantizedWeight:
    """Offline FP4 quantization of a stack of weights w [groups, n_out, k]
    (fp16, CUDA), each with its own tensor scale."""
    _fp16_matrix(w, "w", 3)
    groups, n_out, k = w.shape
    nbytes = int(lib().sharq_weight_bytes_grouped(groups, n_out, k, fmt))
    if nbytes == 0:
        raise SharqError(ERR_INVALID_ARG, f"grouped weight shape {tuple(w.shape)} fmt {fmt}")
    buf = _device_buffer(nbytes, w.device)
    desc = SharqWQ()
    _check(lib().sharq_quantize_weight_grouped(_ptr(w), groups, n_out, k, fmt, _ptr(buf), nbytes, C.byref(desc),
                                               _stream(stream)), "sharq_quantize_weight_grouped")
    return QuantizedWeight(buf, desc)


def group_view(qw: QuantizedWeight, g: int) -> QuantizedWeight:
    """A plain (one-group) descriptor of group g of a stacked weight; it
    shares qw's buffer."""
    d = qw.desc
    _require(0 <= g < max(1, d.groups), f"group {g} out of range (groups = {max(1, d.groups)})")
    stride = weight_bytes(d.n_out, d.k, d.fmt) * g
    v = SharqWQ()
    C.pointer(v)[0] = d
    v.groups = 1
    for f in ("codes", "scales_backbone", "scales_residual", "tensor_scale", "scratch"):
        setattr(v, f, getattr(d, f) + stride)
    return QuantizedWeight(qw.buf, v)


def grouped_rows(rows: int, groups: int) -> int:
    return int(lib().sharq_grouped_rows(rows, groups))


def gather_rows(prep: Prepared, row_idx, offsets: torch.Tensor, rows: int, out: Prepared | None = None,
                stream=None) -> Prepared:
    """Expert-grouped copy of prepared rows: grouped row i of group g (offsets
    [g] <= i < offsets[g+1]) is prepared row row_idx[i] (row_idx None: i).
    row_idx and offsets are int32 CUDA tensors."""
    _int32_vector(offsets, "offsets")
    if row_idx is not None:
        _int32_vector(row_idx, "row_idx")
    _cuda_here(prep.buf, "prep.buf")
    groups = offsets.numel() - 1
    d = prep.desc
    nbytes = int(lib().sharq_gather_bytes(rows, groups, d.k, d.n, d.m, d.fmt))
    if nbytes == 0:
        raise SharqError(ERR_INVALID_ARG, f"gather rows {rows} groups {groups}")
    buf = out.buf if out is not None and out.buf.numel() >= nbytes else _device_buffer(nbytes, prep.buf.device)
    _cuda_here(buf, "out.buf")
    desc = SharqPrep()
    _check(lib().sharq_gather_rows(C.byref(d), _ptr(row_idx), _ptr(offsets), groups, rows, _ptr(buf), buf.numel(),
                                   C.byref(desc), _stream(stream)), "sharq_gather_rows")
    return Prepared(buf, desc)


def prepare_grouped(x: torch.Tensor, offsets: torch.Tensor, ln_w=None, ln_b=None, eps: float = 1e-5, n: int = 2,
                    m: int = 4, fmt: int = NVFP4, norm: str = "layer", out: Prepared | None = None,
                    stream=None) -> Prepared:
    """Preparation of x [rows, k] (fp16, CUDA; rows in grouped order, group g
    = rows offsets[g] .. offsets[g+1]-1) straight into the grouped layout that
    gather_rows writes (equal to gather_rows(prepare(x), None, offsets) in
    codes, scales, metadata and tensor scale). offsets: int32 CUDA tensor."""
    _require(norm in ("layer", "rms") and (norm == "layer" or ln_b is None),
             'norm must be "layer" or "rms" (RMSNorm takes no ln_b)')
    _fp16_matrix(x, "x")
    _int32_vector(offsets, "offsets")
    for t, name in ((ln_w, "ln_w"), (ln_b, "ln_b")):
        if t is not None:
            _fp16_matrix(t.view(-1) if t.is_contiguous() else t, name, 1)
            _require(t.numel() == x.shape[1], f"{name} must have {x.shape[1]} elements")
    rows, k = x.shape
    groups = offsets.numel() - 1
    nbytes = int(lib().sharq_gather_bytes(rows, groups, k, n, m, fmt))
    if nbytes == 0:
        raise SharqError(ERR_INVALID_ARG, f"grouped prep rows {rows} groups {groups} k {k}")
    buf = out.buf if out is not None and out.buf.numel() >= nbytes else _device_buffer(nbytes, x.device)
    _cuda_here(buf, "out.buf")
    desc = SharqPrep()
    _check(lib().sharq_prepare_grouped(_ptr(x) if rows > 0 else None, rows, k, _ptr(offsets), groups, _ptr(ln_w),
                                       _ptr(ln_b), float(eps), 1 if norm == "rms" else 0, n, m, fmt, _ptr(buf),
                                       buf.numel(), C.byref(desc), _stream(stream)), "sharq_prepare_grouped")
    return Prepared(buf, desc)


def linear_grouped(prep: Prepared, offsets: torch.Tensor, qw: QuantizedWeight, rows: int,
                   out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Grouped dual-path FP4 linear: fp16 [rows, n_out] in grouped order,
    group g's rows through group g's weight."""
    _int32_vector(offsets, "offsets")
    _cuda_here(prep.buf, "prep.buf")
    _cuda_here(qw.buf, "qw.buf")
    if out is None:
        out = torch.empty((rows, qw.n_out), dtype=torch.float16, device=prep.buf.device)
    _require(out.dtype == torch.float16 and out.is_contiguous() and tuple(out.shape) == (rows, qw.n_out),
             f"out must be a contiguous fp16 tensor of shape {(rows, qw.n_out)}")
    _cuda_here(out, "out")
    optr = _ptr(out) if out.numel() else None
    _check(lib().sharq_linear_grouped(C.byref(prep.desc), _ptr(offsets), offsets.numel() - 1, rows, C.byref(qw.desc),
                                      optr, _stream(stream)), "sharq_linear_grouped")
    return out


def get_last_error(stream=None) -> int:
    """Synchronizes the stream; returns (and clears) the device status."""
    return int(lib().sharq_get_last_error(_stream(stream)))


def selftest_wait(limit_ns: int, stream=None) -> None:
    """Enqueues the bounded-wait probe (see sharq_selftest_wait)."""
    _check(lib().sharq_selftest_wait(int(limit_ns), _stream(stream)), "sharq_selftest_wait")


def selftest_division(count: int, seed: int = 1, stream=None, examples: bool = False):
    """Mismatches of the encode kernels' division against div.rn (expected 0);
    with examples=True also the first mismatching rows (v, d, q, reference)."""
    out = C.c_uint64(0)
    ex = np.zeros((16, 4), np.float32)
    _check(lib().sharq_selftest_division(int(count), int(seed), C.byref(out), ex.ctypes.data_as(C.c_void_p),
                                         _stream(stream)), "sharq_selftest_division")
    return (int(out.value), ex) if examples else int(out.value)


def last_timeout_site() -> int:
    return int(lib().sharq_last_timeout_site())


def set_wait_limit_ns(ns: int) -> int:
    return int(lib().sharq_set_wait_limit_ns(ns))


def last_launch_count() -> int:
    return int(lib().sharq_last_launch_count())
