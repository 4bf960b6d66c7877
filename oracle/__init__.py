"""Python access to the SharQ CPU oracle (oracle/sharq_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg use it. The CUDA path never imports this package.

Every function takes and returns numpy arrays in the oracle's canonical
layouts (one code per byte, row-major scales, ascending kept indices).
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import numpy as np

from . import build as _build

NVFP4, MXFP4 = 0, 1
BLOCK = {NVFP4: 16, MXFP4: 32}

_lib = None
_omp = False


def use_openmp(on: bool) -> None:
    """Selects the OpenMP build of the same oracle source (independent rows
    and output elements split across threads; identical results) for the
    calls that follow. Default: the single-threaded build."""
    global _lib, _omp
    if bool(on) != _omp:
        _omp = bool(on)
        _lib = None


def threads() -> int:
    """Threads the current build's parallel loops use (1: the plain build)."""
    return int(lib().oracle_threads())


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(_build.build(omp=_omp))
        _declare(_lib)
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _declare(L):
    vp, i64, f32, i32 = C.c_void_p, C.c_int64, C.c_float, C.c_int
    L.oracle_threads.restype = i32
    L.oracle_half_to_double.argtypes = [C.c_uint16]
    L.oracle_half_to_double.restype = C.c_double
    L.oracle_u128_to_double.argtypes = [C.c_uint64, C.c_uint64]
    L.oracle_u128_to_double.restype = C.c_double
    L.oracle_ln_stats.argtypes = [vp, i64, i64, f32, vp, vp]
    L.oracle_rms_stats.argtypes = [vp, i64, i64, f32, vp, vp]
    L.oracle_ln_apply.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp]
    L.oracle_e2m1_value.argtypes = [i32]
    L.oracle_e2m1_value.restype = C.c_double
    L.oracle_e2m1_encode.argtypes = [f32]
    L.oracle_e2m1_encode.restype = i32
    L.oracle_ue4m3_value.argtypes = [i32]
    L.oracle_ue4m3_value.restype = C.c_double
    L.oracle_ue4m3_encode.argtypes = [f32]
    L.oracle_ue4m3_encode.restype = i32
    L.oracle_mx_exponent.argtypes = [f32]
    L.oracle_mx_exponent.restype = i32
    L.oracle_quantize.argtypes = [vp, i64, i64, i32, f32, vp, vp]
    L.oracle_tensor_scale.argtypes = [vp, i64, i32]
    L.oracle_tensor_scale.restype = f32
    L.oracle_mask.argtypes = [vp, i64, i64, i32, i32, vp, vp]
    L.oracle_prepare.argtypes = [vp, i64, i64, vp, vp, f32, i32, i32, i32] + [vp] * 14
    L.oracle_prepare_norm.argtypes = [vp, i64, i64, vp, vp, f32, i32, i32, i32, i32] + [vp] * 14
    L.oracle_quantize_weight.argtypes = [vp, i64, i64, i32, vp, vp, vp, vp]
    L.oracle_linear.argtypes = [vp, vp, vp, vp, f32, vp, vp, f32, i64, i64, i64, i32, vp, vp]
    L.oracle_mask_pairs48.argtypes = [vp, i64, i64, vp, vp]
    L.oracle_double_to_half_rn.argtypes = [C.c_double]
    L.oracle_double_to_half_rn.restype = C.c_uint16
    L.oracle_add_fp16.argtypes = [vp, vp, i64, vp]
    L.oracle_quantize_blk.argtypes = [vp, i64, i64, i32, i32, f32, vp, vp]
    L.oracle_prepare_sparse.argtypes = [vp, i64, i64, vp, vp, f32, i32, i32] + [vp] * 14
    L.oracle_quantize_weight_blk.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, vp]
    L.oracle_linear_blk.argtypes = [vp, vp, i32, vp, vp, i32, f32, vp, vp, i32, f32, i64, i64, i64, i32, vp, vp]


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16
    return a


# ---------------------------------------------------------------------------
# Scalar codecs


def e2m1_encode(y: float) -> int:
    return lib().oracle_e2m1_encode(float(y))


def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code))


def ue4m3_encode(u: float) -> int:
    return lib().oracle_ue4m3_encode(float(u))


def ue4m3_value(code: int) -> float:
    return lib().oracle_ue4m3_value(int(code))


def mx_exponent(a: float) -> int:
    return lib().oracle_mx_exponent(float(a))


def u128_to_double(v: int) -> float:
    return lib().oracle_u128_to_double((v >> 64) & ((1 << 64) - 1), v & ((1 << 64) - 1))


def half_to_double(h: int) -> float:
    return lib().oracle_half_to_double(int(h))


# ---------------------------------------------------------------------------
# Array steps


def ln_stats(x: np.ndarray, eps: float):
    x = _u16(x)
    rows, k = x.shape
    mu = np.empty(rows, np.float32)
    rstd = np.empty(rows, np.float32)
    lib().oracle_ln_stats(_p(x), rows, k, eps, _p(mu), _p(rstd))
    return mu, rstd


def rms_stats(x: np.ndarray, eps: float):
    """RMSNorm statistics: (mu = 0, rstd) per row."""
    x = _u16(x)
    rows, k = x.shape
    mu = np.empty(rows, np.float32)
    rstd = np.empty(rows, np.float32)
    lib().oracle_rms_stats(_p(x), rows, k, eps, _p(mu), _p(rstd))
    return mu, rstd


NORMS = {"layer": 0, "rms": 1}


def ln_apply(x, gamma, beta, mu, rstd):
    x = _u16(x)
    rows, k = x.shape
    g = None if gamma is None else _u16(gamma)
    b = None if beta is None else _u16(beta)
    out = np.empty((rows, k), np.float32)
    lib().oracle_ln_apply(_p(x), rows, k, _p(g), _p(b), _p(np.ascontiguousarray(mu, np.float32)),
                          _p(np.ascontiguousarray(rstd, np.float32)), _p(out))
    return out


def tensor_scale(v: np.ndarray, fmt: int) -> np.float32:
    v = np.ascontiguousarray(v, np.float32)
    return np.float32(lib().oracle_tensor_scale(_p(v), v.size, fmt))


def mask(x_ln: np.ndarray, n: int, m: int):
    x_ln = np.ascontiguousarray(x_ln, np.float32)
    rows, k = x_ln.shape
    idx = np.empty((rows, k // m, n), np.uint8)
    keep = np.empty((rows, k), np.uint8)
    lib().oracle_mask(_p(x_ln), rows, k, n, m, _p(idx), _p(keep))
    return idx, keep


def quantize(v: np.ndarray, fmt: int, s_t: float):
    v = np.ascontiguousarray(v, np.float32)
    rows, k = v.shape
    codes = np.empty((rows, k), np.uint8)
    scales = np.empty((rows, k // BLOCK[fmt]), np.uint8)
    lib().oracle_quantize(_p(v), rows, k, fmt, float(s_t), _p(codes), _p(scales))
    return codes, scales


@dataclass
class Prepared:
    mu: np.ndarray
    rstd: np.ndarray
    x_ln: np.ndarray
    s: np.ndarray
    deq_s: np.ndarray
    r: np.ndarray
    idx: np.ndarray
    keep: np.ndarray
    s_codes: np.ndarray
    s_scales: np.ndarray
    r_codes: np.ndarray
    r_scales: np.ndarray
    s_t: np.float32
    fmt: int
    n: int
    m: int


def prepare(x, gamma, beta, eps: float, n: int, m: int, fmt: int, s_t=None, norm: str = "layer") -> Prepared:
    """The preparation operator on the rows of x. s_t=None derives the
    tensor scale from these rows; a given s_t (the scale of a larger tensor
    these rows were sampled from) is used as is. norm: "layer" (LayerNorm)
    or "rms" (RMSNorm: no centring, beta must be None)."""
    assert norm in NORMS and (norm == "layer" or beta is None)
    x = _u16(x)
    rows, k = x.shape
    blk = BLOCK[fmt]
    g = None if gamma is None else _u16(gamma)
    b = None if beta is None else _u16(beta)
    f = lambda: np.empty((rows, k), np.float32)
    mu, rstd = np.empty(rows, np.float32), np.empty(rows, np.float32)
    x_ln, s, deq_s, r = f(), f(), f(), f()
    idx = np.empty((rows, k // m, n), np.uint8)
    keep = np.empty((rows, k), np.uint8)
    s_codes, r_codes = np.empty((rows, k), np.uint8), np.empty((rows, k), np.uint8)
    s_scales = np.empty((rows, k // blk), np.uint8)
    r_scales = np.empty((rows, k // blk), np.uint8)
    s_t_arr = np.empty(1, np.float32)
    s_t_in = None if s_t is None else np.array([s_t], np.float32)
    lib().oracle_prepare_norm(_p(x), rows, k, _p(g), _p(b), eps, n, m, fmt, NORMS[norm],
                              _p(mu), _p(rstd), _p(x_ln), _p(s), _p(deq_s), _p(r),
                              _p(idx), _p(keep), _p(s_codes), _p(s_scales),
                              _p(r_codes), _p(r_scales), _p(s_t_arr), _p(s_t_in))
    s_t = s_t_arr
    return Prepared(mu, rstd, x_ln, s, deq_s, r, idx, keep, s_codes, s_scales,
                    r_codes, r_scales, s_t[0], fmt, n, m)


@dataclass
class QWeight:
    w_f32: np.ndarray
    codes: np.ndarray
    scales: np.ndarray
    s_tw: np.float32
    fmt: int


def tensor_scale_of(x, gamma, beta, eps: float, fmt: int, norm: str = "layer") -> np.float32:
    """The activation tensor scale over all rows of x (the normalization,
    then amax), computed in row chunks to bound memory."""
    x = _u16(x)
    rows = x.shape[0]
    amax = np.float32(0.0)
    step = max(1, (1 << 24) // max(1, x.shape[1]))
    for r0 in range(0, rows, step):
        xs = x[r0:r0 + step]
        mu, rstd = (ln_stats if norm == "layer" else rms_stats)(xs, eps)
        xl = ln_apply(xs, gamma, beta, mu, rstd)
        amax = max(amax, np.abs(xl).max() if xl.size else np.float32(0))
    if fmt != NVFP4:
        return np.float32(1.0)
    return tensor_scale(np.array([amax], np.float32), fmt)


def quantize_weight(w, fmt: int) -> QWeight:
    w = _u16(w)
    n_out, k = w.shape
    w_f32 = np.empty((n_out, k), np.float32)
    codes = np.empty((n_out, k), np.uint8)
    scales = np.empty((n_out, k // BLOCK[fmt]), np.uint8)
    s_tw = np.empty(1, np.float32)
    lib().oracle_quantize_weight(_p(w), n_out, k, fmt, _p(w_f32), _p(codes), _p(scales), _p(s_tw))
    return QWeight(w_f32, codes, scales, s_tw[0], fmt)


def linear(s_codes, s_scales, r_codes, r_scales, s_t, w_codes, w_scales, s_tw, fmt,
           want_bound: bool = True):
    """fp64 dual-path output and its tolerance scale, for the given rows."""
    s_codes = np.ascontiguousarray(s_codes, np.uint8)
    r_codes = np.ascontiguousarray(r_codes, np.uint8)
    s_scales = np.ascontiguousarray(s_scales, np.uint8)
    r_scales = np.ascontiguousarray(r_scales, np.uint8)
    w_codes = np.ascontiguousarray(w_codes, np.uint8)
    w_scales = np.ascontiguousarray(w_scales, np.uint8)
    rows, k = s_codes.shape
    n_out = w_codes.shape[0]
    out = np.empty((rows, n_out), np.float64)
    bound = np.empty((rows, n_out), np.float64) if want_bound else None
    lib().oracle_linear(_p(s_codes), _p(s_scales), _p(r_codes), _p(r_scales), float(s_t),
                        _p(w_codes), _p(w_scales), float(s_tw), rows, n_out, k, fmt,
                        _p(out), _p(bound))
    return out, bound


def linear_prepared(p: Prepared, qw: QWeight, rows=None):
    """Dual-path output for a Prepared activation (optionally a row subset)."""
    sel = slice(None) if rows is None else rows
    return linear(p.s_codes[sel], p.s_scales[sel], p.r_codes[sel], p.r_scales[sel], p.s_t,
                  qw.codes, qw.scales, qw.s_tw, p.fmt)


# --------------------------------------------------------------------------
# Mixture-of-experts grouped variant. The SharQ abstract names Qwen3-30B-A3B
# (a mixture-of-experts model) among its models without describing the
# expert layers. Reading: each expert's linear is the dual-path linear over
# the rows routed to it; the activation is prepared once over all rows (one
# tensor scale); each expert's weight is quantized on its own.


def expert_of(offsets, i):
    """Group of grouped row i: the g with offsets[g] <= i < offsets[g+1]."""
    offsets = np.asarray(offsets)
    g = int(np.searchsorted(offsets, i, side="right")) - 1
    assert 0 <= g < len(offsets) - 1 and offsets[g] <= i < offsets[g + 1]
    return g


def quantize_weight_grouped(w, fmt: int) -> list:
    """One QWeight per expert; w is [groups][n_out][k]."""
    return [quantize_weight(w[g], fmt) for g in range(w.shape[0])]


def linear_grouped(p: Prepared, row_idx, offsets, qws: list, sel=None, cols=None):
    """out[i] = the dual-path linear of expert g's weight on prepared row
    row_idx[i], for grouped rows i of expert g (offsets[g] <= i <
    offsets[g+1]). sel: grouped rows to compute (default all); cols: output
    columns (default all). Returns (out, bound) like linear()."""
    offsets = np.asarray(offsets)
    row_idx = np.asarray(row_idx)
    sel = np.arange(int(offsets[-1])) if sel is None else np.asarray(sel)
    cols = slice(None) if cols is None else np.asarray(cols)
    n_out = qws[0].codes[cols].shape[0]
    out = np.zeros((len(sel), n_out), np.float64)
    bound = np.zeros((len(sel), n_out), np.float64)
    for j, i in enumerate(sel):
        g = expert_of(offsets, int(i))
        t = int(row_idx[int(i)])
        qw = qws[g]
        o, b = linear(p.s_codes[t:t + 1], p.s_scales[t:t + 1], p.r_codes[t:t + 1], p.r_scales[t:t + 1],
                      p.s_t, qw.codes[cols], qw.scales[cols], qw.s_tw, p.fmt)
        out[j], bound[j] = o[0], b[0]
    return out, bound


# --------------------------------------------------------------------------
# Fused projections and bias. An interface addition: the SharQ abstract
# describes one linear at a time. Reading: a fused weight is its segments
# (q, k, v or gate, up), each quantized on its own with its own tensor
# scale, and the fused output is the segments' outputs side by side. The
# bias (Qwen2.5's q/k/v projections have one) is added after the scaled
# accumulator: out = RN16(RN32(RN32(acc * s_t * s_tW) + b)); here the exact
# fp64 dual-path value plus b.


def quantize_weight_fused(ws, fmt: int) -> list:
    """One QWeight per segment of a fused weight."""
    return [quantize_weight(w, fmt) for w in ws]


def linear_fused(p: Prepared, qws: list, bias=None, rows=None):
    """fp64 output of a fused linear (segments side by side) plus the bias
    (fp16 [n_out] or None), and the tolerance scale: the dual-path bound
    plus |bias|, which bounds |output| and so the final fp16 rounding."""
    parts = [linear_prepared(p, q, rows) for q in qws]
    out = np.concatenate([o for o, _ in parts], axis=1)
    bound = np.concatenate([b for _, b in parts], axis=1)
    if bias is not None:
        b = np.asarray(bias, np.float16).astype(np.float64)
        assert b.shape == (out.shape[1],)
        out = out + b[None, :]
        bound = bound + np.abs(b)[None, :]
    return out, bound


# --------------------------------------------------------------------------
# Pair-wise 4:8 sparse-backbone mode (the pattern the sparse block-scaled FP4
# tensor-core instructions accept). In every aligned group of 8 along K the
# two of the four adjacent pairs with the largest max(|a|, |b|) are kept
# (equal: the lower pair); the backbone and the weights use blocks twice the
# format's length (NVFP4 32, MXFP4 64); the residual keeps the format's own.

SPARSE_BLOCK = {NVFP4: 32, MXFP4: 64}


def mask_pairs48(x_ln: np.ndarray):
    x_ln = np.ascontiguousarray(x_ln, np.float32)
    rows, k = x_ln.shape
    idx = np.empty((rows, k // 8, 4), np.uint8)
    keep = np.empty((rows, k), np.uint8)
    lib().oracle_mask_pairs48(_p(x_ln), rows, k, _p(idx), _p(keep))
    return idx, keep


def quantize_blk(v: np.ndarray, fmt: int, blk: int, s_t: float):
    v = np.ascontiguousarray(v, np.float32)
    rows, k = v.shape
    codes = np.empty((rows, k), np.uint8)
    scales = np.empty((rows, k // blk), np.uint8)
    lib().oracle_quantize_blk(_p(v), rows, k, fmt, blk, float(s_t), _p(codes), _p(scales))
    return codes, scales


def prepare_sparse(x, gamma, beta, eps: float, fmt: int, s_t=None, norm: str = "layer") -> Prepared:
    """The preparation operator in the pair-wise 4:8 mode (n = 4, m = 8 in
    the result; s_scales has one scale per SPARSE_BLOCK[fmt] values)."""
    assert norm in NORMS and (norm == "layer" or beta is None)
    x = _u16(x)
    rows, k = x.shape
    g = None if gamma is None else _u16(gamma)
    b = None if beta is None else _u16(beta)
    f = lambda: np.empty((rows, k), np.float32)
    mu, rstd = np.empty(rows, np.float32), np.empty(rows, np.float32)
    x_ln, s, deq_s, r = f(), f(), f(), f()
    idx = np.empty((rows, k // 8, 4), np.uint8)
    keep = np.empty((rows, k), np.uint8)
    s_codes, r_codes = np.empty((rows, k), np.uint8), np.empty((rows, k), np.uint8)
    s_scales = np.empty((rows, k // SPARSE_BLOCK[fmt]), np.uint8)
    r_scales = np.empty((rows, k // BLOCK[fmt]), np.uint8)
    s_t_arr = np.empty(1, np.float32)
    s_t_in = None if s_t is None else np.array([s_t], np.float32)
    lib().oracle_prepare_sparse(_p(x), rows, k, _p(g), _p(b), eps, fmt, NORMS[norm],
                                _p(mu), _p(rstd), _p(x_ln), _p(s), _p(deq_s), _p(r),
                                _p(idx), _p(keep), _p(s_codes), _p(s_scales),
                                _p(r_codes), _p(r_scales), _p(s_t_arr), _p(s_t_in))
    return Prepared(mu, rstd, x_ln, s, deq_s, r, idx, keep, s_codes, s_scales,
                    r_codes, r_scales, s_t_arr[0], fmt, 4, 8)


def quantize_weight_sparse(w, fmt: int) -> QWeight:
    """Weights for the pair-wise mode: blocks of SPARSE_BLOCK[fmt]."""
    w = _u16(w)
    n_out, k = w.shape
    blk = SPARSE_BLOCK[fmt]
    w_f32 = np.empty((n_out, k), np.float32)
    codes = np.empty((n_out, k), np.uint8)
    scales = np.empty((n_out, k // blk), np.uint8)
    s_tw = np.empty(1, np.float32)
    lib().oracle_quantize_weight_blk(_p(w), n_out, k, fmt, blk, _p(w_f32), _p(codes), _p(scales), _p(s_tw))
    return QWeight(w_f32, codes, scales, s_tw[0], fmt)


def linear_blk(s_codes, s_scales, blk_s, r_codes, r_scales, blk_r, s_t, w_codes, w_scales, blk_w, s_tw, fmt,
               want_bound: bool = True):
    """fp64 dual-path output and its tolerance scale with explicit block
    lengths of the three scale arrays."""
    arr = lambda a: np.ascontiguousarray(a, np.uint8)
    s_codes, r_codes, w_codes = arr(s_codes), arr(r_codes), arr(w_codes)
    s_scales, r_scales, w_scales = arr(s_scales), arr(r_scales), arr(w_scales)
    rows, k = s_codes.shape
    n_out = w_codes.shape[0]
    out = np.empty((rows, n_out), np.float64)
    bound = np.empty((rows, n_out), np.float64) if want_bound else None
    lib().oracle_linear_blk(_p(s_codes), _p(s_scales), blk_s, _p(r_codes), _p(r_scales), blk_r, float(s_t),
                            _p(w_codes), _p(w_scales), blk_w, float(s_tw), rows, n_out, k, fmt,
                            _p(out), _p(bound))
    return out, bound


def linear_sparse(p: Prepared, qw: QWeight, rows=None):
    """Dual-path output for a pair-wise-mode activation and weight."""
    sel = slice(None) if rows is None else rows
    return linear_blk(p.s_codes[sel], p.s_scales[sel], SPARSE_BLOCK[p.fmt], p.r_codes[sel], p.r_scales[sel],
                      BLOCK[p.fmt], p.s_t, qw.codes, qw.scales, SPARSE_BLOCK[p.fmt], qw.s_tw, p.fmt)


# --------------------------------------------------------------------------
# Residual add feeding the preparation operator: x = RN16(h + d) (IEEE
# binary16 addition; in pre-norm transformers the normalization's input is
# the residual stream after this add).


def double_to_half(v: float) -> int:
    """Nearest binary16 (ties to even) of a binary64 value, as bits."""
    return int(lib().oracle_double_to_half_rn(float(v)))


def add_fp16(h, d) -> np.ndarray:
    h, d = _u16(h), _u16(d)
    assert h.shape == d.shape
    x = np.empty(h.shape, np.uint16)
    lib().oracle_add_fp16(_p(h), _p(d), h.size, _p(x))
    return x
