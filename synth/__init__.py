"""Seeded synthetic inputs shared by the CPU oracle, the CUDA path, the tests
and the benchmark.

This module draws random numbers and shapes workloads. It contains none of
SharQ's arithmetic (no LayerNorm, masking, quantization or GEMM), so both sides
of every parity check can consume its bytes without sharing method code.

Generator: counter-based splitmix64 (Steele, Lea & Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014). Draw i of stream (seed, stream)
is mix64(key + (i + 1) * GOLDEN) with key = mix64(seed * GOLDEN ^ stream).
Uniforms take the top 53 bits. Normals come from the Box-Muller transform in
fp64. The bulk generators run in synth.c (OpenMP over independent elements,
so the bytes do not depend on the thread count); the *_np functions state the
same definition in numpy and the tests hold the two equal.

Workloads follow the SharQ abstract ("SharQ: Bridging Activation Sparsity and
FP4 Quantization for LLM Inference", arXiv 2606.26587, abstract): the paper
evaluates Llama-3.1-8B, Qwen2.5-7B and Qwen3-30B-A3B. Their weights are not
used; only the layer shapes are, with outlier-heavy synthetic activations.
"""
from __future__ import annotations

import ctypes as C
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_clib = None


def build(force: bool = False) -> str:
    """Compiles synth.c (the hot loops below) into synth/libsynth.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.run(["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                        _SRC, "-o", _LIB + ".tmp", "-lm"], check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _c():
    global _clib
    if _clib is None:
        L = C.CDLL(build())
        u64, i64, vp = C.c_uint64, C.c_int64, C.c_void_p
        L.synth_normal.argtypes = [u64, u64, i64, i64, vp]
        L.synth_student_fp16.argtypes = [u64, u64, i64, i64, i64, vp, vp]
        L.synth_normal_fp16.argtypes = [u64, u64, i64, i64, i64, vp, vp]
        _clib = L
    return _clib


def _vp(a):
    return a.ctypes.data_as(C.c_void_p)

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK64 = (1 << 64) - 1


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def _key(seed: int, stream: int) -> np.uint64:
    s = np.array([(seed * 0x9E3779B97F4A7C15) & _MASK64], dtype=np.uint64)
    s ^= np.uint64(stream & _MASK64)
    return _mix64(s)[0]


def raw_u64(seed: int, stream: int, count: int, start: int = 0) -> np.ndarray:
    """Draws start .. start+count-1 of the stream, as uint64."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(_key(seed, stream) + idx * GOLDEN)


def uniform(seed: int, stream: int, count: int) -> np.ndarray:
    """U[0, 1) doubles with 53 random bits."""
    return (raw_u64(seed, stream, count) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(seed: int, stream: int, count: int) -> np.ndarray:
    """N(0, 1) doubles by Box-Muller on pairs of uniforms (u1 in (0, 1])."""
    out = np.empty(count, np.float64)
    _c().synth_normal(seed, stream, 0, count, _vp(out))
    return out


def normal_np(seed: int, stream: int, count: int) -> np.ndarray:
    """Pure-numpy statement of normal(), kept as the reference of synth.c."""
    pairs = (count + 1) // 2
    u = uniform(seed, stream, 2 * pairs)
    u1 = 1.0 - u[0::2]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    th = (2.0 * math.pi) * u2
    out = np.empty(2 * pairs, dtype=np.float64)
    out[0::2] = r * np.cos(th)
    out[1::2] = r * np.sin(th)
    return out[:count]


def student_t3_np(seed: int, stream: int, count: int) -> np.ndarray:
    """Student-t with 3 degrees of freedom: Z / sqrt((Z1^2 + Z2^2 + Z3^2) / 3)
    (pure-numpy reference of synth.c)."""
    z = normal_np(seed, stream, 4 * count).reshape(count, 4)
    chi = (z[:, 1] ** 2 + z[:, 2] ** 2 + z[:, 3] ** 2) / 3.0
    return z[:, 0] / np.sqrt(chi)


def permutation(seed: int, stream: int, n: int) -> np.ndarray:
    """A seeded permutation of range(n) (argsort of random keys, stable)."""
    return np.argsort(raw_u64(seed, stream, n), kind="stable")


def to_fp16(v: np.ndarray) -> np.ndarray:
    """Clamp to the fp16 finite range, then round to nearest even."""
    return np.clip(v, -65504.0, 65504.0).astype(np.float16)


# Stream identifiers: one stream per tensor role, so tensors never share draws.
S_BODY, S_OUTLIER_PICK, S_OUTLIER_GAIN, S_WEIGHT, S_GATE, S_LN = 1, 2, 3, 4, 5, 6


def gaussian_gains(seed: int, k: int, n_outlier: int, gain: float) -> np.ndarray:
    g = np.ones(k, np.float64)
    g[permutation(seed, S_OUTLIER_PICK, k)[:n_outlier]] = gain
    return g


def student_gains(seed: int, k: int, outlier_frac: float = 0.01, gain_lo: float = 20.0,
                  gain_hi: float = 100.0) -> np.ndarray:
    n_out = int(math.ceil(outlier_frac * k))
    g = np.ones(k, np.float64)
    g[permutation(seed, S_OUTLIER_PICK, k)[:n_out]] = gain_lo + (gain_hi - gain_lo) * uniform(seed, S_OUTLIER_GAIN, n_out)
    return g


def activations_gaussian(seed: int, rows: int, k: int, n_outlier: int, gain: float, row0: int = 0) -> np.ndarray:
    """X ~ N(0, 1) with n_outlier channels (seeded choice) multiplied by gain.
    Rows row0 .. row0+rows-1 of the tensor of that seed."""
    out = np.empty((rows, k), np.uint16)
    _c().synth_normal_fp16(seed, S_BODY, row0, rows, k, _vp(gaussian_gains(seed, k, n_outlier, gain)), _vp(out))
    return out.view(np.float16)


def activations_student(seed: int, rows: int, k: int, outlier_frac: float = 0.01,
                        gain_lo: float = 20.0, gain_hi: float = 100.0, row0: int = 0) -> np.ndarray:
    """Student-t(3) body; ceil(outlier_frac * k) channels, fixed across tokens,
    scaled by a per-channel gain drawn from U[gain_lo, gain_hi]. Rows row0 ..
    row0+rows-1 of the tensor of that seed."""
    out = np.empty((rows, k), np.uint16)
    g = student_gains(seed, k, outlier_frac, gain_lo, gain_hi)
    _c().synth_student_fp16(seed, S_BODY, row0, rows, k, _vp(g), _vp(out))
    return out.view(np.float16)


def activations_student_np(seed: int, rows: int, k: int, outlier_frac: float = 0.01,
                           gain_lo: float = 20.0, gain_hi: float = 100.0) -> np.ndarray:
    """Pure-numpy statement of activations_student (reference of synth.c)."""
    x = student_t3_np(seed, S_BODY, rows * k).reshape(rows, k)
    x *= student_gains(seed, k, outlier_frac, gain_lo, gain_hi)[None, :]
    return to_fp16(x)


def weights(seed: int, n_out: int, k: int, std: float = 0.02, row0: int = 0) -> np.ndarray:
    """W ~ N(0, std^2), fp16, [n_out, k] row-major (K-major)."""
    out = np.empty((n_out, k), np.uint16)
    _c().synth_normal_fp16(seed, S_WEIGHT, row0, n_out, k, _vp(np.full(k, std)), _vp(out))
    return out.view(np.float16)


def ln_params(seed: int, k: int) -> tuple[np.ndarray, np.ndarray]:
    """Non-trivial LayerNorm gamma ~ 1 + 0.1 N(0,1), beta ~ 0.1 N(0,1), fp16."""
    g = normal(seed, S_LN, 2 * k)
    return to_fp16(1.0 + 0.1 * g[:k]), to_fp16(0.1 * g[k:])


def moe_routing(seed: int, tokens: int, n_experts: int, top_k: int):
    """Top-k routing from N(0,1) gate logits (softmax is monotone, so top-k of
    the logits is top-k of the probabilities); ties go to the lower expert.

    Returns (row_idx, expert_offsets): for expert e, the token indices routed
    to it are row_idx[expert_offsets[e]:expert_offsets[e+1]], ascending.
    """
    logits = normal(seed, S_GATE, tokens * n_experts).reshape(tokens, n_experts)
    order = np.argsort(-logits, axis=1, kind="stable")[:, :top_k]
    counts = np.zeros(n_experts, dtype=np.int64)
    lists = [[] for _ in range(n_experts)]
    for t in range(tokens):
        for e in order[t]:
            lists[int(e)].append(t)
    offsets = np.zeros(n_experts + 1, dtype=np.int32)
    for e in range(n_experts):
        counts[e] = len(lists[e])
        offsets[e + 1] = offsets[e] + counts[e]
    row_idx = np.concatenate([np.asarray(l, dtype=np.int32) for l in lists]) if tokens else np.zeros(0, np.int32)
    return row_idx.astype(np.int32), offsets


# --------------------------------------------------------------------------
# Workload shapes


@dataclass(frozen=True)
class Linear:
    name: str
    k: int       # input features
    n_out: int   # output features
    prep: str    # which prepared activation feeds it


@dataclass(frozen=True)
class LayerSet:
    """One transformer layer's linears. Linears that read the same activation
    share one preparation (q/k/v share one, gate/up share one)."""
    name: str
    hidden: int
    preps: tuple          # (prep name, k)
    linears: tuple        # Linear entries


LLAMA31_8B = LayerSet(
    name="llama3.1-8b",
    hidden=4096,
    preps=(("attn_in", 4096), ("o_in", 4096), ("mlp_in", 4096), ("down_in", 14336)),
    linears=(
        Linear("q_proj", 4096, 4096, "attn_in"),
        Linear("k_proj", 4096, 1024, "attn_in"),
        Linear("v_proj", 4096, 1024, "attn_in"),
        Linear("o_proj", 4096, 4096, "o_in"),
        Linear("gate_proj", 4096, 14336, "mlp_in"),
        Linear("up_proj", 4096, 14336, "mlp_in"),
        Linear("down_proj", 14336, 4096, "down_in"),
    ),
)

QWEN25_7B = LayerSet(
    name="qwen2.5-7b",
    hidden=3584,
    preps=(("attn_in", 3584), ("o_in", 3584), ("mlp_in", 3584), ("down_in", 18944)),
    linears=(
        Linear("q_proj", 3584, 3584, "attn_in"),
        Linear("k_proj", 3584, 512, "attn_in"),
        Linear("v_proj", 3584, 512, "attn_in"),
        Linear("o_proj", 3584, 3584, "o_in"),
        Linear("gate_proj", 3584, 18944, "mlp_in"),
        Linear("up_proj", 3584, 18944, "mlp_in"),
        Linear("down_proj", 18944, 3584, "down_in"),
    ),
)

# Qwen3-30B-A3B MoE FFN: hidden 2048, 128 experts of intermediate 768, top-8.
QWEN3_MOE = dict(hidden=2048, inter=768, n_experts=128, top_k=8)


def layer_seeds(index: int) -> tuple[int, int]:
    """Activation seed and weight seed of the index-th tensor of a layer set."""
    return index, 1000 + index
