#!/usr/bin/env python
"""Benchmark of the SharQ per-linear-layer hot path on B200.

One step = the whole hot path over one batch: the 4 preparation operators and
the 7 dual-path FP4 linears of a Llama-3.1-8B-shaped layer set
(q/k/v share one prep, gate/up share one prep) on M tokens, NVFP4, 2:4.
Inputs are seeded synthetic Student-t(3) activations with 1% outlier channels
scaled x20..100 and N(0, 0.02^2) weights (quantized offline, outside the
timed region), resident in HBM. L2 is flushed (256 MB write) before every
timed step; each step is timed with CUDA events on the launching stream.

Prints ONE JSON line (rank 0). Multi-GPU: one process per GPU (torchrun),
each rank runs its own replica of the workload (the path has no exchange
step), value = all ranks' tokens / the max over ranks of the timed region.

--impl reference times the CPU oracle (oracle/) on a bounded sample of the
same workload, as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "SharQ linear tokens/s & FP4 TFLOPS (% tensor peak), prep GB/s (% HBM)"
UNIT = "tokens/s"
EPS = 1e-5
N_KEEP, M_GROUP = 2, 4
FP4_OVER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor throughput on B200 (9 / 2.25 PFLOP/s)


def prep_bytes_per_elem(fmt, n, m, dense_s=False):
    """Algorithmic bytes per activation element of one preparation: x read
    (2), the backbone's codes compressed to its n of every m values
    (0.5 n / m), the mask metadata (n indices of ceil(log2 m) bits per m),
    one scale byte per block for S and for R (1/16 NVFP4, 1/32 MXFP4) and
    the residual's codes (0.5). NVFP4 2:4: 3.0 B. dense_s=True counts the
    backbone's codes as stored by the dense-backbone layout (0.5, zeros off
    the mask): NVFP4 2:4 3.25 B."""
    meta = n * max(1, (m - 1).bit_length()) / m / 8.0
    s_codes = 0.5 if dense_s else 0.5 * n / m
    return 2 + s_codes + meta + 2.0 / (16 if fmt == 0 else 32) + 0.5


PREP_BYTES_PER_ELEM = prep_bytes_per_elem(0, N_KEEP, M_GROUP)  # 3.0
PREP_BYTES_PER_ELEM_DENSE_S = prep_bytes_per_elem(0, N_KEEP, M_GROUP, dense_s=True)  # 3.25
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) of the 7 GEMM launches of one M = 8192 step:
# the sum over the step's linears of dram__bytes_read.sum +
# dram__bytes_write.sum of one ncu capture per shape (one launch each, caches
# flushed before it: q and o 70.9 MB, k and v 40.7 MB, gate and up 277.8 MB,
# down 248.5 MB) of the current dual_gemm_kernel. Set to None whenever the
# kernel changes until it is captured again.
GEMM_TRAFFIC_BYTES_PER_STEP_M8192 = 1027.6e6
# The only performance and accuracy figures of the method's own evaluation
# (abstract of "SharQ: Bridging Activation Sparsity and FP4 Quantization for
# LLM Inference"): other hardware and end-to-end serving, reported for
# context next to the measured line, never as its baseline.
PAGES_CONTEXT = {
    "hardware": "RTX 5090 (sm_120)",
    "latency_vs_fp16": "2.2-2.4x lower",
    "throughput_vs_fp8": "1.2-1.4x higher",
    "accuracy_gap_recovered": "43-63% of the NVFP4-to-FP16 gap",
    "comparable": "no: other GPU, whole-model serving; see quality for this path's output error",
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["sharq", "reference"], default="sharq")
    ap.add_argument("--tokens", type=int, default=8192, help="M: tokens per step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-quality", action="store_true", help="skip the output-error report")
    ap.add_argument("--cpu-sample-tokens", type=int, default=1)
    ap.add_argument("--cpu-sample-cols", type=int, default=8192,
                    help="output columns of each linear in the CPU sample (cost is linear in columns)")
    ap.add_argument("--ref-sample-cols", type=int, default=1024,
                    help="output columns of each linear in each step of the reference arm's sample")
    ap.add_argument("--no-extras", action="store_true", help="skip the other workloads' summary numbers")
    ap.add_argument("--case", default=None,
                    help="time one op instead of the layer set: prep:M:K[:fmt:n:m] or linear:M:N:K[:fmt:n:m] "
                         "(fmt 0 = NVFP4, 1 = MXFP4); used for profiling and shape sweeps")
    ap.add_argument("--outlier-frac", type=float, default=0.01)
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(tokens):
    return (f"Llama-3.1-8B layer set (q/k/v 4096->4096/1024/1024, o 4096->4096, gate/up 4096->14336, "
            f"down 14336->4096): 4 preps + 7 dual-path linears, M={tokens} tokens, NVFP4, 2:4")


def layer_set():
    ls = synth.LLAMA31_8B
    preps = list(ls.preps)
    return ls, preps


def flops_algorithmic(tokens):
    ls, _ = layer_set()
    return sum(2.0 * tokens * l.n_out * l.k * (1.0 + N_KEEP / M_GROUP) for l in ls.linears)


def flops_executed(tokens):
    ls, _ = layer_set()
    return sum(4.0 * tokens * l.n_out * l.k for l in ls.linears)  # both paths run dense FP4 MMAs


def prep_bytes_algorithmic(tokens):
    _, preps = layer_set()
    return sum(PREP_BYTES_PER_ELEM * tokens * k for _, k in preps)


# ---------------------------------------------------------------------------
# Clock sampling during the timed region


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu_index = gpu_index
        self.path = os.path.join(tempfile.gettempdir(), f"sharq_clocks_{os.getpid()}.csv")

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", str(self.gpu_index)], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self, t_start: float, t_end: float):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].isdigit():
                    rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [int(r[1]) for r in rows]
        loaded = [r for r in rows if r[3] not in ("[N/A]",) and _float(r[3]) > 200.0] or rows
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in loaded:
            for name, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(statistics.median(int(r[1]) for r in loaded)), "sm_max_mhz": float(max(int(r[2]) for r in rows)),
                "reasons": sorted(reasons), "samples": len(loaded), "sm_mhz_min": min(sm)}


def _float(s):
    try:
        return float(s)
    except ValueError:
        return 0.0


# ---------------------------------------------------------------------------
# Distributed plumbing


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "sharq" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# The CUDA path


def run_sharq(args, world, rank, local):
    import sparsity_gemm_b200 as sq
    from sparsity_gemm_b200 import build as lib_build
    if not os.path.exists(sq.LIB_PATH):
        lib_build.build()
    sq.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    M = args.tokens
    ls, preps = layer_set()
    prep_index = {name: i for i, (name, _) in enumerate(preps)}

    # Inputs: seeded synthetic activations and weights, resident in HBM.
    xs_host = [torch.from_numpy(synth.activations_student(i, M, k).view(np.float16)) for i, (_, k) in enumerate(preps)]
    xs = [t.to(dev) for t in xs_host]
    qws = []
    for j, lin in enumerate(ls.linears):
        w = torch.from_numpy(synth.weights(1000 + j, lin.n_out, lin.k).view(np.float16)).to(dev)
        qws.append(sq.quantize_weight(w, sq.NVFP4))
        del w
    prep_bufs = [sq.prepare(xs[i], None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4) for i in range(len(preps))]
    outs = [torch.empty((M, lin.n_out), dtype=torch.float16, device=dev) for lin in ls.linears]
    torch.cuda.synchronize()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    launches = [0]

    def step(x_list, ev=None):
        for i in range(len(preps)):
            prep_bufs[i] = sq.prepare(x_list[i], None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4, out=prep_bufs[i])
            launches[0] += sq.last_launch_count()
            if ev is not None:
                ev[1 + i].record(stream)
        for j, lin in enumerate(ls.linears):
            sq.linear(prep_bufs[prep_index[lin.prep]], qws[j], out=outs[j])
            launches[0] += sq.last_launch_count()
            if ev is not None:
                ev[1 + len(preps) + j].record(stream)

    n_ev = 1 + len(preps) + len(ls.linears)
    for _ in range(args.warmup):
        flush.zero_()
        step(xs)
    torch.cuda.synchronize()
    status = sq.get_last_error()
    if status != sq.OK:
        raise RuntimeError(f"device status after warm-up: {sq.status_name(status)}")

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    launches[0] = 0
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0 = time.time()
        for s in range(args.steps):
            flush.zero_()
            events[s][0].record(stream)
            step(xs, events[s])
        torch.cuda.synchronize()
        t1 = time.time()
    barrier(world)
    status = sq.get_last_error()
    if status != sq.OK:
        raise RuntimeError(f"device status after timing: {sq.status_name(status)}")

    prep_ms = gemm_ms = 0.0
    gemm_each = np.zeros(len(ls.linears))
    for ev in events:
        for i in range(len(preps)):
            prep_ms += ev[i].elapsed_time(ev[i + 1])
        for j in range(len(ls.linears)):
            d = ev[len(preps) + j].elapsed_time(ev[len(preps) + j + 1])
            gemm_ms += d
            gemm_each[j] += d
    total_ms = prep_ms + gemm_ms
    total_ms_max = max_over_ranks(total_ms, world, dev)
    steps = args.steps
    value = world * M * steps / (total_ms_max / 1e3)
    gpu_launches = launches[0]

    peaks, peak_src = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    gemm_alg_tflops = flops_algorithmic(M) * steps / (gemm_ms / 1e3) / 1e12
    gemm_exec_tflops = flops_executed(M) * steps / (gemm_ms / 1e3) / 1e12
    prep_gbs = prep_bytes_algorithmic(M) * steps / (prep_ms / 1e3) / 1e9

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": args.warmup,
        "ms_per_step": total_ms_max / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 + ue4m3/16 + fp32 tensor scale), fp32 accumulate",
        "data": "synthetic (seeded Student-t(3) activations, 1% outlier channels x20-100; N(0,0.02^2) weights)",
        "config": {"workload": workload_desc(M), "tokens": M, "fmt": "nvfp4", "nm": f"{N_KEEP}:{M_GROUP}",
                   "layernorm": "gamma/beta NULL", "l2": "flushed (256 MB write) before every timed step",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "kernel": "dual_gemm_kernel (7 linears)",
                     "achieved": gemm_alg_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": gemm_alg_tflops / fp4_peak,
                     "traffic": GEMM_TRAFFIC_BYTES_PER_STEP_M8192 if M == 8192 else None,
                     "traffic_scope": "DRAM bytes of the 7 GEMM launches of one step (sum of per-launch ncu captures)",
                     "peak_source": f"{peak_src} bf16 {peaks['bf16_tflops']} TF/s x {FP4_OVER_BF16} (FP4/BF16 nominal)",
                     "flops_per_step": flops_algorithmic(M), "flop_count": "2*M*N*K*(1+n/m)",
                     "executed_tflops": gemm_exec_tflops, "executed_frac": gemm_exec_tflops / fp4_peak},
        "prep_roofline": {"bound": "hbm", "kernel": "ln_stats_warp_kernel + prep_encode_kernel (4 preps)",
                          "achieved": prep_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                          "frac": prep_gbs / peaks["hbm_gbs"], "bytes_per_elem": PREP_BYTES_PER_ELEM,
                          "bytes_count": "algorithmic: x 2 + S codes 0.25 (n/m of 0.5) + metadata 0.125 + "
                                         "S scales 0.0625 + R codes 0.5 + R scales 0.0625",
                          "dense_s": {"bytes_per_elem": PREP_BYTES_PER_ELEM_DENSE_S,
                                      "achieved": prep_gbs * PREP_BYTES_PER_ELEM_DENSE_S / PREP_BYTES_PER_ELEM,
                                      "frac": prep_gbs * PREP_BYTES_PER_ELEM_DENSE_S / PREP_BYTES_PER_ELEM
                                      / peaks["hbm_gbs"],
                                      "note": "S codes as the dense-backbone layout stores them (0.5 B)"}},
        "split_ms_per_step": {"prep": prep_ms / steps, "gemm": gemm_ms / steps,
                              "gemm_each": {lin.name: float(gemm_each[j] / steps) for j, lin in enumerate(ls.linears)}},
        "gpu_launches": gpu_launches,
        "wall_s_timed": t1 - t0,
        "pages_context": PAGES_CONTEXT,
    }
    cs = clocks.summary(t0, t1)
    result["clocks"] = {"sm_mhz": cs.get("sm_mhz"), "sm_max_mhz": cs.get("sm_max_mhz"), "reasons": cs.get("reasons"),
                        "samples": cs.get("samples")}

    if not args.no_quality and rank == 0:
        result["quality"] = quality_report(sq, dev, xs, preps, prep_bufs, outs, ls, prep_index)
    if not args.no_e2e:
        result["e2e"] = e2e_sharq(args, sq, dev, stream, xs_host, preps, prep_bufs, qws, outs, ls, prep_index, world)
    if rank == 0 and world == 1 and not args.no_extras:
        result["configs"] = config_summaries(args)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args)
    return result


E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def dequantized_weight(sq, qw, dev):
    """deq(Q(W)) in fp32 from the library's exported codes and scales (for
    the quality report only): E2M1 value x block scale x tensor scale."""
    wx = sq.weight_export(qw)
    blk = sq.BLOCK[qw.desc.fmt]
    codes = torch.from_numpy(wx["codes"]).to(dev).long()
    sc = torch.from_numpy(wx["scales"]).to(dev)
    sv = (sc.view(torch.float8_e4m3fn).float() if qw.desc.fmt == sq.NVFP4
          else torch.exp2(sc.float() - 127.0))
    table = torch.tensor(E2M1_VALUES, device=dev)
    return table[codes] * sv.repeat_interleave(blk, dim=1) * float(wx["s_tw"])


def quality_report(sq, dev, xs, preps, prep_bufs, outs, ls, prep_index):
    """Output error of every linear against an fp16 GEMM, next to plain NVFP4
    (reported, not gated). Reference: RN16(LayerNorm(x)) times the fp16
    weight, in fp32 (torch, outside the timed region: a measuring stick, not
    part of the path). Plain NVFP4: this library with n = m (the mask keeps
    everything) and the residual codes zeroed, so that only deq(Q(X_ln))
    times deq(Q(W)) remains. Metric: relative Frobenius error; "recovered"
    is the share of plain NVFP4's error that SharQ removes. Both paths use
    the same Q(W), whose error dominates against the fp16 weight, so the
    report adds the activation-side error: against RN16(LayerNorm(x)) times
    deq(Q(W))."""
    torch.backends.cuda.matmul.allow_tf32 = False
    per = {}
    plain = {}
    for i, (name, k) in enumerate(preps):
        p = sq.prepare(xs[i], None, None, EPS, M_GROUP, M_GROUP, sq.NVFP4)
        off = p.desc.r_codes - p.buf.data_ptr()
        p.buf[off:off + xs[i].shape[0] * k // 2].zero_()
        plain[name] = p
    for j, lin in enumerate(ls.linears):
        i = prep_index[lin.prep]
        w = torch.from_numpy(synth.weights(1000 + j, lin.n_out, lin.k).view(np.float16)).to(dev)
        x_ln = torch.nn.functional.layer_norm(xs[i].float(), (lin.k,), eps=EPS).half().float()
        qw = sq.quantize_weight(w, sq.NVFP4)
        out_plain = sq.linear(plain[lin.prep], qw)
        rec = {}
        for tag, wref in (("", w.float()), ("act_", None)):
            ref = x_ln @ (wref if wref is not None else dequantized_weight(sq, qw, dev)).t()
            nref = torch.linalg.vector_norm(ref).item()
            e_sharq = torch.linalg.vector_norm(outs[j].float() - ref).item() / nref
            e_plain = torch.linalg.vector_norm(out_plain.float() - ref).item() / nref
            rec.update({tag + "sharq": e_sharq, tag + "nvfp4": e_plain, tag + "recovered": (e_plain - e_sharq) / e_plain})
            del ref
        per[lin.name] = rec
        del x_ln, out_plain, qw, w
    torch.cuda.synchronize()
    st = sq.get_last_error()
    if st != sq.OK:
        raise RuntimeError(f"device status after quality report: {sq.status_name(st)}")
    return {"metric": "relative Frobenius error vs fp16 GEMM of RN16(LayerNorm(x)) W^T",
            "plain": "NVFP4 (n = m, no residual path)",
            "mean_sharq": float(np.mean([v["sharq"] for v in per.values()])),
            "mean_nvfp4": float(np.mean([v["nvfp4"] for v in per.values()])),
            "mean_recovered": float(np.mean([v["recovered"] for v in per.values()])),
            "act_reference": "RN16(LayerNorm(x)) deq(Q(W))^T: activation-side error only",
            "mean_act_sharq": float(np.mean([v["act_sharq"] for v in per.values()])),
            "mean_act_nvfp4": float(np.mean([v["act_nvfp4"] for v in per.values()])),
            "mean_act_recovered": float(np.mean([v["act_recovered"] for v in per.values()])),
            "per_linear": per}


def e2e_sharq(args, sq, dev, stream, xs_host, preps, prep_bufs, qws, outs, ls, prep_index, world):
    """Same metric through the public API with host buffers: every step copies
    its activations from pinned host memory and reads every output back. The
    steps are pipelined as a serving loop would run them: inputs go in on a
    copy stream one step ahead (two device input buffers), each linear's
    output goes back on a second copy stream as soon as it is computed (two
    device output sets), so host-to-device copies, compute and
    device-to-host copies overlap; events order every buffer reuse. The
    timed region runs from the first input copy to the completion of the
    last output copy."""
    M = args.tokens
    steps = max(3, min(args.steps, 20))
    pinned_in = [t.pin_memory() for t in xs_host]
    dev_in = [[torch.empty_like(t, device=dev) for t in xs_host] for _ in range(2)]
    dev_out = [outs, [torch.empty_like(o) for o in outs]]
    pinned_out = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs] for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()

    def run(n_steps, e_start=None):
        in_ready = [ev() for _ in range(n_steps)]
        in_free = [ev() for _ in range(n_steps)]      # compute of step s no longer reads dev_in[s % 2]
        lin_done = [[ev() for _ in outs] for _ in range(n_steps)]
        out_free = [ev() for _ in range(n_steps)]     # outputs of step s copied back
        if e_start is not None:
            e_start.record(s_in)

        def load(t):
            with torch.cuda.stream(s_in):
                if t >= 2:
                    s_in.wait_event(in_free[t - 2])
                for i, x in enumerate(pinned_in):
                    dev_in[t % 2][i].copy_(x, non_blocking=True)
                in_ready[t].record(s_in)

        load(0)
        for t in range(n_steps):
            if t + 1 < n_steps:
                load(t + 1)
            b = t % 2
            stream.wait_event(in_ready[t])
            if t >= 2:
                stream.wait_event(out_free[t - 2])
            for i in range(len(preps)):
                prep_bufs[i] = sq.prepare(dev_in[b][i], None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4,
                                          out=prep_bufs[i], stream=stream)
            in_free[t].record(stream)
            for j, lin in enumerate(ls.linears):
                sq.linear(prep_bufs[prep_index[lin.prep]], qws[j], out=dev_out[b][j], stream=stream)
                lin_done[t][j].record(stream)
            with torch.cuda.stream(s_out):
                for j in range(len(outs)):
                    s_out.wait_event(lin_done[t][j])
                    pinned_out[b][j].copy_(dev_out[b][j], non_blocking=True)
                out_free[t].record(s_out)
        return out_free[n_steps - 1]

    run(2)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    last = run(steps, e_start=e0)
    s_out.wait_event(last)
    e1.record(s_out)
    torch.cuda.synchronize()
    st = sq.get_last_error()
    if st != sq.OK:
        raise RuntimeError(f"device status after the end-to-end run: {sq.status_name(st)}")
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return {"value": world * M * steps / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(sum(t.numel() * 2 for t in xs_host)),
            "d2h_bytes_per_step": int(sum(o.numel() * 2 for o in outs)), "steps": steps,
            "pipelined": "inputs one step ahead and outputs back on separate copy streams"}


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)


def oracle_sample(tokens: int, cols: int):
    """Builds the bounded CPU sample: `tokens` rows of each activation and the
    first `cols` output columns of each linear (weights quantized up front)."""
    import oracle
    ls, preps = layer_set()
    xs = [synth.activations_student(i, tokens, k) for i, (_, k) in enumerate(preps)]
    ws = []
    for j, lin in enumerate(ls.linears):
        c = min(cols, lin.n_out)
        ws.append(oracle.quantize_weight(synth.weights(1000 + j, c, lin.k), oracle.NVFP4))
    return ls, preps, xs, ws


def oracle_step(sample):
    """One pass of the oracle over the sample; returns the linears' outputs."""
    import oracle
    ls, preps, xs, ws = sample
    prepared = [oracle.prepare(x, None, None, EPS, N_KEEP, M_GROUP, oracle.NVFP4) for x in xs]
    pidx = {name: i for i, (name, _) in enumerate(preps)}
    return [oracle.linear_prepared(prepared[pidx[lin.prep]], ws[j])[0] for j, lin in enumerate(ls.linears)]


def token_fraction(sample, tokens):
    """Token-equivalents of one sample step: the sample runs the full prep of
    `tokens` rows but only a fraction of each linear's columns; the linears
    dominate the oracle's cost, so weight them by their share of the MACs."""
    ls, preps, xs, ws = sample
    macs_full = sum(l.n_out * l.k for l in ls.linears)
    macs_sample = sum(w.codes.shape[0] * l.k for w, l in zip(ws, ls.linears))
    return tokens * macs_sample / macs_full


def _host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(args):
    """The oracle on the host cores, on a bounded sample of the step: the
    single-threaded build on one core, then the OpenMP build of the same
    source on all cores (independent rows and output elements split across
    threads), whose outputs are checked equal to the single-threaded ones."""
    import oracle
    sample = oracle_sample(args.cpu_sample_tokens, args.cpu_sample_cols)
    oracle.use_openmp(False)
    t0 = time.perf_counter()
    out1 = oracle_step(sample)
    dt1 = time.perf_counter() - t0
    tok = token_fraction(sample, args.cpu_sample_tokens)
    oracle.use_openmp(True)
    threads = oracle.threads()
    t0 = time.perf_counter()
    out_n = oracle_step(sample)
    dtn = time.perf_counter() - t0
    oracle.use_openmp(False)
    same = all(np.array_equal(a, b) for a, b in zip(out1, out_n))
    desc = (f"{args.cpu_sample_tokens} token(s): full prep of each activation row, and the first "
            f"{args.cpu_sample_cols} output columns of each linear (cost linear in columns; value = "
            f"{tok:.4f} token-equivalents / time)")
    return {"value": tok / dt1, "unit": UNIT, "cores": 1, "kind": "oracle", "nproc": _host_cores(),
            "sample": desc + f", single-threaded C oracle: {dt1:.2f} s",
            "all_cores": {"value": tok / dtn, "unit": UNIT, "cores": threads, "seconds": dtn,
                          "build": "same source with OpenMP over independent rows and output elements",
                          "outputs_identical": bool(same)}}


def config_summaries(args):
    """Summary numbers of the other workloads, measured after the timed step
    (each on its own, L2 flushed before every step): the preparation with the
    normalization's parameters (LayerNorm gamma/beta, RMSNorm weight; the
    timed step takes none), the pair-wise 4:8 sparse-backbone mode on the
    same layer set, the Qwen2.5-7B layer set (NVFP4/MXFP4 x 2:4/4:8, M =
    4096), the Qwen3-30B-A3B MoE FFN (M = 4096) and the decode-vs-prefill
    sweep of the down projection (1% outliers)."""
    peaks, _ = load_peaks()
    st, wu = 5, 2
    M = args.tokens
    ls = synth.LLAMA31_8B
    out = {"steps": st, "warmup": wu, "timing": "median per step, CUDA events, L2 flushed before every step"}
    keep = ("tokens_per_s", "ms_per_step", "prep_ms", "gemm_ms", "gemm_tflops", "gemm_frac", "gemm_executed_frac",
            "prep_gbs", "prep_frac", "prep_bytes_per_elem")
    pick = lambda r: {k: r[k] for k in ("fmt", "nm") + keep}
    aff = {}
    for name, a in (("layernorm_gamma_beta", "layer"), ("rmsnorm_weight", "rms")):
        prep_ms, gemm_ms = time_layer_set(ls, M, 0, N_KEEP, M_GROUP, st, wu, affine=a)
        aff[name] = pick(layer_set_report(ls, M, 0, N_KEEP, M_GROUP, prep_ms, gemm_ms, peaks))
    out["llama31_8b_prep_with_norm_params"] = aff
    prep_ms, gemm_ms = time_layer_set(ls, M, 0, N_KEEP, M_GROUP, st, wu, sparse=True)
    out["llama31_8b_pairwise_sparse_backbone"] = layer_set_report(ls, M, 0, N_KEEP, M_GROUP, prep_ms, gemm_ms,
                                                                  peaks, sparse=True)
    q = []
    for fmt in (0, 1):
        for n, m in ((2, 4), (4, 8)):
            prep_ms, gemm_ms = time_layer_set(synth.QWEN25_7B, 4096, fmt, n, m, st, wu)
            q.append(pick(layer_set_report(synth.QWEN25_7B, 4096, fmt, n, m, prep_ms, gemm_ms, peaks)))
    out["qwen25_7b_m4096"] = q
    a = argparse.Namespace(**vars(args))
    a.steps, a.warmup, a.outlier_frac = 10, 3, 0.01
    moe = run_moe(a, 4096)
    out["qwen3_30b_a3b_moe_m4096"] = {k: moe[k] for k in ("tokens_per_s", "ms_per_step", "rows", "padded_rows", "ms",
                                                           "fused_gate_up")}
    out["qwen3_30b_a3b_moe_m4096"]["grouped_gemm_frac"] = moe["gemm_roofline"]["frac"]
    dec = run_decode(a, 1)
    out["llama31_8b_decode_m1"] = {
        "graph_us_per_step": dec["graph_ms_per_step"] * 1e3,
        "fused_projections_graph_us_per_step": dec["fused_projections"]["graph_ms_per_step"] * 1e3,
        "weight_stream_floor_us": dec["weight_stream_floor_ms"] * 1e3,
        "graph_frac_of_floor": dec["graph_frac_of_floor"],
        "fused_frac_of_floor": dec["fused_projections"]["graph_frac_of_floor"],
        "launch": "CUDA graph replay, 4 preps + 7 linears (fused: 4 + 4), L2 flushed before every step"}
    sw = run_sweep(a, [1, 16, 256, 2048, 16384])
    out["down_proj_decode_prefill_sweep"] = {
        "crossover_M": sw["crossover_M"],
        "rows": [{k: r[k] for k in ("M", "prep_us", "gemm_us", "gemm_tflops", "gemm_bound", "gemm_roofline_frac")}
                 for r in sw["rows"]]}
    torch.cuda.empty_cache()
    return out


def run_reference(args, world, rank):
    if rank != 0:
        return None
    sample = oracle_sample(args.cpu_sample_tokens, args.ref_sample_cols)
    for _ in range(args.warmup):
        oracle_step(sample)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(sample)
        times.append(time.perf_counter() - t0)
    tok = token_fraction(sample, args.cpu_sample_tokens)
    total = sum(times)
    value = tok * len(times) / total
    desc = (f"{args.cpu_sample_tokens} token(s) per step: full prep of each activation row and the first "
            f"{args.ref_sample_cols} output columns of each linear ({tok:.4f} token-equivalents per step)")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / len(times) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 prep, f64 GEMM",
            "data": "synthetic (same seeded generator)",
            "config": {"workload": workload_desc(args.tokens), "tokens": args.tokens, "fmt": "nvfp4",
                       "nm": f"{N_KEEP}:{M_GROUP}"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
                             "nproc": _host_cores()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def run_case(args, world, rank, local):
    """One op on one shape: W warm-up and K timed launches, L2 flushed before
    each, CUDA events on the launching stream. Prints a JSON line with the
    op's time and its roofline figure."""
    import sparsity_gemm_b200 as sq
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    parts = args.case.split(":")
    kind = parts[0]
    nums = [int(v) for v in parts[1:]]
    peaks, peak_src = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    if kind == "moe":
        return run_moe(args, nums[0] if nums else 4096)
    if kind == "sweep":
        return run_sweep(args)
    if kind == "vendor_fp4":
        return run_vendor_fp4(args)
    if kind == "fused":
        return run_fused(args, nums[0] if nums else 8192)
    if kind == "decode":
        return run_decode(args, nums[0] if nums else 1)
    if kind == "add_prep":
        return run_add_prep(args, *(nums[:2] if len(nums) >= 2 else [8192, 4096]))
    if kind == "sparse":
        return run_sparse(args, nums[0] if nums else 8192)
    if kind == "qwen25":
        return run_qwen25(args, nums[0] if nums else 4096)
    if kind == "layerset":
        return run_layerset_tokens(args, nums or [1, 16, 128, 2048, 8192])
    if kind == "prep":
        M, K = nums[:2]
        fmt, n, m = (nums[2:5] + [0, N_KEEP, M_GROUP][len(nums[2:5]):])
        x = torch.from_numpy(synth.activations_student(0, M, K, outlier_frac=args.outlier_frac).view(np.float16)).to(dev)
        buf = sq.prepare(x, None, None, EPS, n, m, fmt)
        op = lambda: sq.prepare(x, None, None, EPS, n, m, fmt, out=buf)
        per_elem = prep_bytes_per_elem(fmt, n, m)
        work, unit, peak, bound = per_elem * M * K, "GB/s", peaks["hbm_gbs"], "hbm"
    elif kind == "prep_sparse":
        M, K = nums[:2]
        fmt = nums[2] if len(nums) > 2 else 0
        x = torch.from_numpy(synth.activations_student(0, M, K, outlier_frac=args.outlier_frac).view(np.float16)).to(dev)
        buf = sq.prepare_sparse(x, None, None, EPS, fmt)
        op = lambda: sq.prepare_sparse(x, None, None, EPS, fmt, out=buf)
        work, unit, peak, bound = prep_bytes_per_elem_sparse(fmt) * M * K, "GB/s", peaks["hbm_gbs"], "hbm"
    elif kind == "linear_sparse":
        M, N, K = nums[:3]
        fmt = nums[3] if len(nums) > 3 else 0
        x = torch.from_numpy(synth.activations_student(0, M, K, outlier_frac=args.outlier_frac).view(np.float16)).to(dev)
        w = torch.from_numpy(synth.weights(1000, N, K).view(np.float16)).to(dev)
        qw = sq.quantize_weight_sparse(w, fmt)
        prep = sq.prepare_sparse(x, None, None, EPS, fmt)
        out = torch.empty((M, N), dtype=torch.float16, device=dev)
        op = lambda: sq.linear(prep, qw, out=out)
        work, unit, bound = 3.0 * M * N * K, "TFLOP/s", "tensor"
        peak = peaks["bf16_tflops"] * FP4_OVER_BF16 * 1e3  # in GFLOP/s, scaled below
    elif kind == "linear":
        M, N, K = nums[:3]
        fmt, n, m = (nums[3:6] + [0, N_KEEP, M_GROUP][len(nums[3:6]):])
        x = torch.from_numpy(synth.activations_student(0, M, K, outlier_frac=args.outlier_frac).view(np.float16)).to(dev)
        w = torch.from_numpy(synth.weights(1000, N, K).view(np.float16)).to(dev)
        qw = sq.quantize_weight(w, fmt)
        prep = sq.prepare(x, None, None, EPS, n, m, fmt)
        out = torch.empty((M, N), dtype=torch.float16, device=dev)
        op = lambda: sq.linear(prep, qw, out=out)
        work, unit, bound = 2.0 * M * N * K * (1.0 + n / m), "TFLOP/s", "tensor"
        peak = peaks["bf16_tflops"] * FP4_OVER_BF16 * 1e3  # in GFLOP/s, scaled below
    else:
        raise SystemExit(f"unknown case {args.case}")
    for _ in range(args.warmup):
        flush.zero_()
        op()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        op()
        b.record(stream)
    torch.cuda.synchronize()
    st = sq.get_last_error()
    if st != sq.OK:
        raise RuntimeError(sq.status_name(st))
    ms = [a.elapsed_time(b) for a, b in evs]
    t = statistics.median(ms) / 1e3
    achieved = work / t / 1e9  # GB/s or GFLOP/s
    if unit == "TFLOP/s":
        achieved /= 1e3
        peak /= 1e3
    return {"case": args.case, "ms_median": t * 1e3, "ms_min": min(ms), "achieved": achieved, "unit": unit,
            "peak": peak, "frac": achieved / peak, "bound": bound, "steps": args.steps,
            "outlier_frac": args.outlier_frac, "peak_source": peak_src}


def fused_linears(ls):
    """The layer set's linears grouped by the activation they read (q/k/v,
    o, gate/up, down): one fused linear per group, in order."""
    groups = []
    for lin in ls.linears:
        if groups and groups[-1][0].prep == lin.prep:
            groups[-1].append(lin)
        else:
            groups.append([lin])
    return groups


def run_fused(args, M):
    """The layer-set step with the linears that share an input fused (q/k/v
    into one weight, gate/up into one; each segment keeps its own tensor
    scale, so the outputs equal the separate linears'): 4 preps + 4 linears,
    timed like the default step. Per-linear event times included."""
    import sparsity_gemm_b200 as sq
    dev = torch.device("cuda", torch.cuda.current_device())
    ls, preps = layer_set()
    prep_index = {name: i for i, (name, _) in enumerate(preps)}
    groups = fused_linears(ls)
    xs = [torch.from_numpy(synth.activations_student(i, M, k).view(np.float16)).to(dev)
          for i, (_, k) in enumerate(preps)]
    lin_index = {lin.name: j for j, lin in enumerate(ls.linears)}
    qws = []
    for g in groups:
        ws = [torch.from_numpy(synth.weights(1000 + lin_index[l.name], l.n_out, l.k).view(np.float16)).to(dev)
              for l in g]
        qws.append(sq.quantize_weight_fused(ws, sq.NVFP4) if len(ws) > 1 else sq.quantize_weight(ws[0], sq.NVFP4))
        del ws
    bufs = [sq.prepare(xs[i], None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4) for i in range(len(preps))]
    outs = [torch.empty((M, q.n_out), dtype=torch.float16, device=dev) for q in qws]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    n_ev = 1 + len(preps) + len(groups)

    def step(ev=None):
        for i in range(len(preps)):
            bufs[i] = sq.prepare(xs[i], None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4, out=bufs[i])
            if ev is not None:
                ev[1 + i].record(stream)
        for j, g in enumerate(groups):
            sq.linear(bufs[prep_index[g[0].prep]], qws[j], out=outs[j])
            if ev is not None:
                ev[1 + len(preps) + j].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    for s in range(args.steps):
        flush.zero_()
        events[s][0].record(stream)
        step(events[s])
    torch.cuda.synchronize()
    st = sq.get_last_error()
    if st != sq.OK:
        raise RuntimeError(sq.status_name(st))
    prep_ms = sum(ev[i].elapsed_time(ev[i + 1]) for ev in events for i in range(len(preps))) / args.steps
    each = [sum(ev[len(preps) + j].elapsed_time(ev[len(preps) + j + 1]) for ev in events) / args.steps
            for j in range(len(groups))]
    total = prep_ms + sum(each)
    return {"case": args.case, "tokens_per_s": M / (total / 1e3), "ms_per_step": total, "prep_ms": prep_ms,
            "gemm_ms": sum(each), "gemm_each": {"+".join(l.name for l in g): each[j] for j, g in enumerate(groups)},
            "steps": args.steps}


def prep_bytes_per_elem_sparse(fmt):
    """Algorithmic bytes per element of the pair-wise 4:8 mode's preparation:
    x (2), the kept half of the backbone codes (0.25), 4 metadata bits per 8
    values (0.0625), one backbone scale per 32 (64) values, the residual's
    codes (0.5) and one residual scale per 16 (32) values. NVFP4: 2.90625 B."""
    blk = 16 if fmt == 0 else 32
    return 2 + 0.25 + 0.0625 + 1.0 / (2 * blk) + 0.5 + 1.0 / blk


def time_layer_set(ls, M, fmt, n, m, steps, warmup, sparse=False, affine=None):
    """Event timing of one layer set's step (its preps, then its linears) at
    M tokens with L2 flushed before every step: medians of the per-step prep
    and GEMM milliseconds. sparse: the pair-wise 4:8 mode (n, m ignored).
    affine: None, "layer" (LayerNorm gamma/beta) or "rms" (RMSNorm weight)."""
    import sparsity_gemm_b200 as sq
    dev = torch.device("cuda", torch.cuda.current_device())
    preps = list(ls.preps)
    prep_index = {name: i for i, (name, _) in enumerate(preps)}
    xs = [torch.from_numpy(synth.activations_student(i, M, k).view(np.float16)).to(dev)
          for i, (_, k) in enumerate(preps)]
    qws = []
    for j, lin in enumerate(ls.linears):
        w = torch.from_numpy(synth.weights(1000 + j, lin.n_out, lin.k).view(np.float16)).to(dev)
        qws.append(sq.quantize_weight_sparse(w, fmt) if sparse else sq.quantize_weight(w, fmt))
        del w
    lnp = []
    for i, (_, k) in enumerate(preps):
        g = b = None
        if affine is not None:
            g16, b16 = synth.ln_params(50 + i, k)
            g = torch.from_numpy(g16.view(np.float16)).to(dev)
            b = torch.from_numpy(b16.view(np.float16)).to(dev) if affine == "layer" else None
        lnp.append((g, b))
    norm = "rms" if affine == "rms" else "layer"

    def prep_one(i, out=None):
        g, b = lnp[i]
        if sparse:
            return sq.prepare_sparse(xs[i], g, b, EPS, fmt, out=out, norm=norm)
        return sq.prepare(xs[i], g, b, EPS, n, m, fmt, out=out, norm=norm)

    bufs = [prep_one(i) for i in range(len(preps))]
    outs = [torch.empty((M, lin.n_out), dtype=torch.float16, device=dev) for lin in ls.linears]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    np_ = len(preps)

    def step(ev=None):
        for i in range(np_):
            prep_one(i, bufs[i])
        if ev is not None:
            ev[1].record(stream)
        for j, lin in enumerate(ls.linears):
            sq.linear(bufs[prep_index[lin.prep]], qws[j], out=outs[j])

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for ev in evs:
        flush.zero_()
        ev[0].record(stream)
        step(ev)
        ev[2].record(stream)
    torch.cuda.synchronize()
    st = sq.get_last_error()
    if st != sq.OK:
        raise RuntimeError(sq.status_name(st))
    prep_ms = statistics.median([e[0].elapsed_time(e[1]) for e in evs])
    gemm_ms = statistics.median([e[1].elapsed_time(e[2]) for e in evs])
    del xs, qws, bufs, outs, flush
    torch.cuda.empty_cache()
    return prep_ms, gemm_ms


def layer_set_report(ls, M, fmt, n, m, prep_ms, gemm_ms, peaks, sparse=False):
    """Throughput and roofline figures of one layer-set timing. The GEMM's
    algorithmic FLOPs are 2 M N K (1 + n/m); executed FLOPs count what the
    tensor cores run in dense-MMA units: both paths dense (4 M N K) in the
    default mode, half of K on the backbone in the pair-wise mode (3 M N K,
    equal to the algorithmic count)."""
    if sparse:
        n, m = 4, 8
    flops = sum(2.0 * M * l.n_out * l.k * (1.0 + n / m) for l in ls.linears)
    executed = sum((3.0 if sparse else 4.0) * M * l.n_out * l.k for l in ls.linears)
    per_elem = prep_bytes_per_elem_sparse(fmt) if sparse else prep_bytes_per_elem(fmt, n, m)
    pbytes = sum(per_elem * M * k for _, k in ls.preps)
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    gemm_tf = flops / (gemm_ms / 1e3) / 1e12
    exec_tf = executed / (gemm_ms / 1e3) / 1e12
    prep_gbs = pbytes / (prep_ms / 1e3) / 1e9
    return {"tokens": M, "fmt": "nvfp4" if fmt == 0 else "mxfp4", "nm": "pair-wise 4:8" if sparse else f"{n}:{m}",
            "backbone_mma": "tcgen05.mma.sp on the K-compacted backbone" if sparse else "dense MMA, zeros off the mask",
            "tokens_per_s": M / ((prep_ms + gemm_ms) / 1e3), "ms_per_step": prep_ms + gemm_ms,
            "prep_ms": prep_ms, "gemm_ms": gemm_ms, "gemm_tflops": gemm_tf, "gemm_frac": gemm_tf / fp4_peak,
            "gemm_executed_tflops": exec_tf, "gemm_executed_frac": exec_tf / fp4_peak,
            "prep_gbs": prep_gbs, "prep_frac": prep_gbs / peaks["hbm_gbs"], "prep_bytes_per_elem": per_elem}


def run_add_prep(args, M, K):
    """The residual add x = h + d followed by the preparation of x, fused
    (sharq_prepare_add: x's statistics taken in the add's pass, so the encode
    pass is the only other read of x) and unfused (the add, then
    sharq_prepare, which reads x twice). The unfused add is torch's fp16 add
    (context for the comparison only; the library has no standalone add).
    Bytes: the add moves 6 B per element (h, d in, x out); the preparation's
    algorithmic 3.0 B per element counts its own read of x."""
    import sparsity_gemm_b200 as sq
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    h = torch.from_numpy(synth.activations_student(0, M, K).view(np.float16)).to(dev)
    d = torch.from_numpy(synth.activations_student(1, M, K, outlier_frac=0.0).view(np.float16)).to(dev)
    x = torch.empty_like(h)
    buf = sq.prepare(h, None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def fused():
        sq.prepare_add(h, d, None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4, x_out=x, out=buf)

    def unfused():
        torch.add(h, d, out=x)
        sq.prepare(x, None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4, out=buf)

    res = {}
    for name, op in (("fused", fused), ("unfused", unfused)):
        for _ in range(args.warmup):
            flush.zero_()
            op()
        ms = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            op()
            b.record(stream)
            b.synchronize()
            ms.append(a.elapsed_time(b))
        t = statistics.median(ms) / 1e3
        nbytes = (6.0 + PREP_BYTES_PER_ELEM - 2.0) * M * K  # add (6) + prep without its own read of x
        res[name] = {"us": t * 1e6, "algorithmic_gbs": nbytes / t / 1e9, "frac": nbytes / t / 1e9 / peaks["hbm_gbs"]}
    st = sq.get_last_error()
    if st != sq.OK:
        raise RuntimeError(sq.status_name(st))
    return {"case": args.case, "M": M, "K": K, "fmt": "nvfp4", "nm": f"{N_KEEP}:{M_GROUP}", **res,
            "bytes_per_elem": 6.0 + PREP_BYTES_PER_ELEM - 2.0,
            "bytes_count": "add: h, d read and x written (6); preparation outputs (1.0): 7.0 B per element",
            "peak_source": peak_src, "l2": "flushed (256 MB write) before every call", "steps": args.steps}


def run_sparse(args, M):
    """The Llama-3.1-8B layer set at M tokens (8192 by default), NVFP4, in the
    default mode (element-wise 2:4, dense backbone MMA) and the pair-wise 4:8
    mode (structured-sparse backbone MMA), and MXFP4 in the pair-wise mode."""
    peaks, peak_src = load_peaks()
    rows = []
    for fmt, sparse in ((0, False), (0, True), (1, True)):
        prep_ms, gemm_ms = time_layer_set(synth.LLAMA31_8B, M, fmt, N_KEEP, M_GROUP, args.steps, args.warmup,
                                          sparse=sparse)
        rows.append(layer_set_report(synth.LLAMA31_8B, M, fmt, N_KEEP, M_GROUP, prep_ms, gemm_ms, peaks, sparse))
    return {"case": args.case, "workload": workload_desc(M), "rows": rows,
            "peak_source": f"{peak_src}: FP4 = bf16 {peaks['bf16_tflops']} TF/s x {FP4_OVER_BF16}, "
            f"HBM {peaks['hbm_gbs']} GB/s", "l2": "flushed (256 MB write) before every step", "steps": args.steps}


def run_qwen25(args, M):
    """The Qwen2.5-7B layer set (hidden 3584, GQA kv 512, intermediate 18944)
    at M tokens (prefill, 4096 by default) for each format and N:M ratio:
    {NVFP4, MXFP4} x {2:4, 4:8}."""
    peaks, peak_src = load_peaks()
    rows = []
    for fmt in (0, 1):
        for n, m in ((2, 4), (4, 8)):
            prep_ms, gemm_ms = time_layer_set(synth.QWEN25_7B, M, fmt, n, m, args.steps, args.warmup)
            rows.append(layer_set_report(synth.QWEN25_7B, M, fmt, n, m, prep_ms, gemm_ms, peaks))
    return {"case": args.case, "workload": "Qwen2.5-7B layer set (q/k/v 3584->3584/512/512, o 3584->3584, "
            "gate/up 3584->18944, down 18944->3584): 4 preps + 7 dual-path linears", "tokens": M, "rows": rows,
            "peak_source": f"{peak_src}: FP4 = bf16 {peaks['bf16_tflops']} TF/s x {FP4_OVER_BF16}, "
            f"HBM {peaks['hbm_gbs']} GB/s", "l2": "flushed (256 MB write) before every step", "steps": args.steps}


def run_layerset_tokens(args, tokens):
    """The Llama-3.1-8B layer set (NVFP4, 2:4) at each token count (decode to
    prefill: 1, 16, 128, 2048, 8192 by default)."""
    peaks, peak_src = load_peaks()
    rows = []
    for M in tokens:
        prep_ms, gemm_ms = time_layer_set(synth.LLAMA31_8B, M, 0, N_KEEP, M_GROUP, args.steps, args.warmup)
        rows.append(layer_set_report(synth.LLAMA31_8B, M, 0, N_KEEP, M_GROUP, prep_ms, gemm_ms, peaks))
    return {"case": args.case, "workload": workload_desc("M"), "rows": rows,
            "peak_source": f"{peak_src}: FP4 = bf16 {peaks['bf16_tflops']} TF/s x {FP4_OVER_BF16}, "
            f"HBM {peaks['hbm_gbs']} GB/s", "l2": "flushed (256 MB write) before every step",
            "launch": "eager from Python (see --case decode:M for CUDA-graph replay)", "steps": args.steps}


def run_decode(args, M):
    """The layer-set step at decode sizes (M tokens, default 1): 4 preps + 7
    linears launched eagerly from Python, and the same step captured once in
    a CUDA graph and replayed. L2 is flushed before every step (outside the
    graph), so the weights stream from HBM as they do when a model's layers
    take turns; the roofline is that weight stream (codes + scales of the 7
    weights) at the measured HBM bandwidth. Also timed (graph only): the
    fused-projection layout a serving stack uses, q/k/v as one weight and
    gate/up as one (quantize_weight_fused, each segment with its own tensor
    scale): 4 preps + 4 linears, the same weight bytes."""
    import sparsity_gemm_b200 as sq
    dev = torch.device("cuda", torch.cuda.current_device())
    ls, preps = layer_set()
    prep_index = {name: i for i, (name, _) in enumerate(preps)}
    xs = [torch.from_numpy(synth.activations_student(i, M, k).view(np.float16)).to(dev)
          for i, (_, k) in enumerate(preps)]
    qws = []
    for j, lin in enumerate(ls.linears):
        w = torch.from_numpy(synth.weights(1000 + j, lin.n_out, lin.k).view(np.float16)).to(dev)
        qws.append(sq.quantize_weight(w, sq.NVFP4))
        del w
    bufs = [sq.prepare(xs[i], None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4) for i in range(len(preps))]
    outs = [torch.empty((M, lin.n_out), dtype=torch.float16, device=dev) for lin in ls.linears]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peaks, peak_src = load_peaks()

    def step():
        for i in range(len(preps)):
            sq.prepare(xs[i], None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4, out=bufs[i])
        for j, lin in enumerate(ls.linears):
            sq.linear(bufs[prep_index[lin.prep]], qws[j], out=outs[j])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(max(args.warmup, 1)):
            step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager_out = [o.clone() for o in outs]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    stream = torch.cuda.current_stream()

    def timed(run):
        for _ in range(args.warmup):
            flush.zero_()
            run()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            run()
            b.record(stream)
        torch.cuda.synchronize()
        return statistics.median([a.elapsed_time(b) for a, b in ev])

    eager_ms = timed(step)
    graph_ms = timed(graph.replay)
    same = all(torch.equal(o.view(torch.int16), e.view(torch.int16)) for o, e in zip(outs, eager_out))

    # fused projections: q/k/v and gate/up, each group one weight
    groups = {}
    for j, lin in enumerate(ls.linears):
        groups.setdefault(lin.prep, []).append(j)
    fqws, fouts, fprep = [], [], []
    for prep_name, idx in groups.items():
        ws = [torch.from_numpy(synth.weights(1000 + j, ls.linears[j].n_out, ls.linears[j].k).view(np.float16)).to(dev)
              for j in idx]
        fqws.append(sq.quantize_weight_fused(ws, sq.NVFP4) if len(ws) > 1 else sq.quantize_weight(ws[0], sq.NVFP4))
        del ws
        fouts.append(torch.empty((M, sum(ls.linears[j].n_out for j in idx)), dtype=torch.float16, device=dev))
        fprep.append(prep_index[prep_name])

    def fused_step():
        for i in range(len(preps)):
            sq.prepare(xs[i], None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4, out=bufs[i])
        for g in range(len(fqws)):
            sq.linear(bufs[fprep[g]], fqws[g], out=fouts[g])

    with torch.cuda.stream(side):
        for _ in range(max(args.warmup, 1)):
            fused_step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    fgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(fgraph):
        fused_step()
    fused_ms = timed(fgraph.replay)
    # the fused outputs against the separate linears' (equal up to the fp32
    # summation order: a different split-K factor changes it)
    fused_same, fused_diff = True, 0.0
    for g, (prep_name, idx) in enumerate(groups.items()):
        c = 0
        for j in idx:
            n = ls.linears[j].n_out
            a, b = fouts[g][:, c:c + n].float(), outs[j].float()
            fused_same &= torch.equal(fouts[g][:, c:c + n].view(torch.int16), outs[j].view(torch.int16))
            fused_diff = max(fused_diff, float(((a - b).abs() / b.abs().clamp_min(1e-3)).max()))
            c += n
    st = sq.get_last_error()
    if st != sq.OK:
        raise RuntimeError(sq.status_name(st))
    w_bytes = sum(l.n_out * l.k / 2 + l.n_out * l.k / 16 for l in ls.linears)  # E2M1 codes + UE4M3 scales
    x_bytes = sum(M * k * 2 for _, k in preps)
    floor_ms = (w_bytes + x_bytes) / (peaks["hbm_gbs"] * 1e9) * 1e3
    return {"case": args.case, "tokens": M, "eager_ms_per_step": eager_ms, "graph_ms_per_step": graph_ms,
            "graph_tokens_per_s": M / (graph_ms / 1e3), "kernels_per_step": 4 * 2 + 7,
            "weight_stream_floor_ms": floor_ms, "graph_frac_of_floor": floor_ms / graph_ms,
            "graph_equals_eager": same,
            "fused_projections": {"layout": "q/k/v one weight, gate/up one weight: 4 preps + 4 linears",
                                  "graph_ms_per_step": fused_ms, "graph_tokens_per_s": M / (fused_ms / 1e3),
                                  "graph_frac_of_floor": floor_ms / fused_ms, "bits_equal_separate": bool(fused_same),
                                  "max_rel_diff_vs_separate": fused_diff}, "peak_source": f"{peak_src} hbm {peaks['hbm_gbs']} GB/s",
            "l2": "flushed (256 MB write) before every step", "steps": args.steps}


def run_sweep(args, ms=None):
    """Decode-vs-prefill sweep on the Llama-3.1-8B down projection (14336 ->
    4096), NVFP4 2:4: for M = 1, 2, 4, ..., 16384 the prep and the dual GEMM
    are timed separately (CUDA events, L2 flushed before every call, median
    of the steps). Reported per M: prep GB/s (algorithmic bytes), GEMM
    TFLOP/s (algorithmic), GEMM GB/s over the weight and activation bytes it
    must read, and which roofline bounds it (t_ideal = max(flops / FP4 peak,
    bytes / HBM peak))."""
    import sparsity_gemm_b200 as sq
    dev = torch.device("cuda", torch.cuda.current_device())
    K, N = 14336, 4096
    peaks, peak_src = load_peaks()
    fp4 = peaks["bf16_tflops"] * FP4_OVER_BF16 * 1e12
    hbm = peaks["hbm_gbs"] * 1e9
    w = torch.from_numpy(synth.weights(1006, N, K).view(np.float16)).to(dev)
    qw = sq.quantize_weight(w, sq.NVFP4)
    del w
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    w_bytes = N * K * (0.5 + 1.0 / 16)
    rows = []
    for M in (ms or [1 << lg for lg in range(15)]):
        x = torch.from_numpy(synth.activations_student(6, M, K, outlier_frac=args.outlier_frac).view(np.float16)).to(dev)
        p = sq.prepare(x, None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4)
        out = torch.empty((M, N), dtype=torch.float16, device=dev)
        ops = (lambda: sq.prepare(x, None, None, EPS, N_KEEP, M_GROUP, sq.NVFP4, out=p),
               lambda: sq.linear(p, qw, out=out))
        t = []
        for op in ops:
            for _ in range(args.warmup):
                flush.zero_()
                op()
            ms = []
            for _ in range(args.steps):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                op()
                b.record(stream)
                b.synchronize()
                ms.append(a.elapsed_time(b))
            t.append(statistics.median(ms) / 1e3)
        st = sq.get_last_error()
        if st != sq.OK:
            raise RuntimeError(sq.status_name(st))
        flops = 2.0 * M * N * K * (1 + N_KEEP / M_GROUP)
        g_bytes = w_bytes + M * K * (1.0 + 2.0 / 16) + 2.0 * M * N
        t_ideal = max(flops / fp4, g_bytes / hbm)
        rows.append({"M": M, "prep_us": t[0] * 1e6, "prep_gbs": PREP_BYTES_PER_ELEM * M * K / t[0] / 1e9,
                     "gemm_us": t[1] * 1e6, "gemm_tflops": flops / t[1] / 1e12, "gemm_gbs": g_bytes / t[1] / 1e9,
                     "gemm_bound": "tensor" if flops / fp4 > g_bytes / hbm else "hbm",
                     "gemm_roofline_frac": t_ideal / t[1]})
        del x, p, out
    cross = next((r["M"] for r in rows if r["gemm_bound"] == "tensor"), None)
    return {"case": "sweep", "workload": "Llama-3.1-8B down projection 14336 -> 4096, NVFP4 2:4, M = 1 .. 16384",
            "outlier_frac": args.outlier_frac, "crossover_M": cross,
            "peaks": {"fp4_tflops": fp4 / 1e12, "hbm_gbs": hbm / 1e9, "source": peak_src},
            "l2": "flushed (256 MB write) before every call", "steps": args.steps, "rows": rows}


def run_vendor_fp4(args):
    """Context only, outside the library: the vendor's NVFP4 GEMM (cuBLASLt
    through torch._scaled_mm, random FP4 codes, unit scales) on the layer
    set's GEMM shapes, timed with CUDA events (L2 flushed before each call).
    One dense FP4 GEMM per call; the dual-path linear runs two such
    contractions (backbone and residual) per call."""
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rows = []

    def ones_blocked(r, c):
        return torch.ones(((r + 127) // 128 * 128) * ((c + 3) // 4 * 4), device=dev).to(torch.float8_e4m3fn)

    for (M, N, K) in [(8192, 4096, 14336), (8192, 14336, 4096), (8192, 4096, 4096), (8192, 1024, 4096)]:
        g = torch.Generator(device=dev).manual_seed(0)
        a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g).view(torch.float4_e2m1fn_x2)
        b = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g).view(torch.float4_e2m1fn_x2)
        sa, sb = ones_blocked(M, K // 16), ones_blocked(N, K // 16)
        f = lambda: torch._scaled_mm(a, b.t(), sa, sb, out_dtype=torch.bfloat16)
        for _ in range(args.warmup):
            flush.zero_()
            f()
        ms = []
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            f()
            e1.record()
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        t = statistics.median(ms) / 1e3
        rows.append({"M": M, "N": N, "K": K, "us": t * 1e6, "tflops": 2.0 * M * N * K / t / 1e12})
    return {"case": "vendor_fp4", "what": "cuBLASLt NVFP4 GEMM via torch._scaled_mm, one dense contraction per call",
            "l2": "flushed (256 MB write) before every call", "steps": args.steps, "rows": rows}


def run_moe(args, tokens):
    """The Qwen3-30B-A3B-shaped MoE FFN (hidden 2048, 128 experts of
    intermediate 768, top-8 routing from N(0,1) gate logits) as one step:
    prep of the token activation, expert-grouped gather, gate and up
    grouped linears, prep of the down projection's grouped-order input
    straight into the grouped layout, down grouped linear. L2 flushed before every
    step; every launch timed with CUDA events on the launching stream."""
    import sparsity_gemm_b200 as sq
    dev = torch.device("cuda", torch.cuda.current_device())
    cfg = synth.QWEN3_MOE
    hidden, inter, groups, top_k = cfg["hidden"], cfg["inter"], cfg["n_experts"], cfg["top_k"]
    fmt, n, m = 0, N_KEEP, M_GROUP
    peaks, peak_src = load_peaks()
    row_idx, offsets = synth.moe_routing(0, tokens, groups, top_k)
    rows = len(row_idx)
    h16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.float16)).to(dev)
    x = h16(synth.activations_student(0, tokens, hidden, outlier_frac=args.outlier_frac))
    xd = h16(synth.activations_student(1, rows, inter, outlier_frac=args.outlier_frac))
    ri = torch.from_numpy(row_idx).to(dev)
    off = torch.from_numpy(offsets).to(dev)
    qws = {}
    for j, (name, n_out, k) in enumerate([("gate", inter, hidden), ("up", inter, hidden), ("down", hidden, inter)]):
        w = h16(np.stack([synth.weights(2000 + 1000 * j + g, n_out, k) for g in range(groups)]))
        qws[name] = sq.quantize_weight_grouped(w, fmt)
        del w
    p_tok = sq.prepare(x, None, None, EPS, n, m, fmt)
    g_tok = sq.gather_rows(p_tok, ri, off, rows)
    g_d = sq.prepare_grouped(xd, off, None, None, EPS, n, m, fmt)
    o_gate = torch.empty((rows, inter), dtype=torch.float16, device=dev)
    o_up = torch.empty_like(o_gate)
    o_down = torch.empty((rows, hidden), dtype=torch.float16, device=dev)
    ops = [
        ("prep", lambda: sq.prepare(x, None, None, EPS, n, m, fmt, out=p_tok)),
        ("gather", lambda: sq.gather_rows(p_tok, ri, off, rows, out=g_tok)),
        ("gate", lambda: sq.linear_grouped(g_tok, off, qws["gate"], rows, out=o_gate)),
        ("up", lambda: sq.linear_grouped(g_tok, off, qws["up"], rows, out=o_up)),
        ("prep_down", lambda: sq.prepare_grouped(xd, off, None, None, EPS, n, m, fmt, out=g_d)),
        ("down", lambda: sq.linear_grouped(g_d, off, qws["down"], rows, out=o_down)),
    ]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    launches = 0
    for i in range(args.warmup):
        flush.zero_()
        for _, f in ops:
            f()
            launches += sq.last_launch_count() if i == 0 else 0
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ops) + 1)] for _ in range(args.steps)]
    for e in ev:
        flush.zero_()
        e[0].record(stream)
        for i, (_, f) in enumerate(ops):
            f()
            e[i + 1].record(stream)
    torch.cuda.synchronize()
    st = sq.get_last_error()
    if st != sq.OK:
        raise RuntimeError(sq.status_name(st))
    per = {name: statistics.median([e[i].elapsed_time(e[i + 1]) for e in ev]) for i, (name, _) in enumerate(ops)}
    step_ms = statistics.median([e[0].elapsed_time(e[-1]) for e in ev])

    # gate and up stacked into one grouped weight per expert ([2 * inter,
    # hidden], one tensor scale per expert): one grouped linear reads each
    # expert's activation tiles once for both projections
    w = h16(np.stack([np.concatenate([synth.weights(2000 + g, inter, hidden), synth.weights(3000 + g, inter, hidden)])
                      for g in range(groups)]))
    q_gu = sq.quantize_weight_grouped(w, fmt)
    del w
    o_gu = torch.empty((rows, 2 * inter), dtype=torch.float16, device=dev)
    gu = lambda: sq.linear_grouped(g_tok, off, q_gu, rows, out=o_gu)
    for _ in range(args.warmup):
        flush.zero_()
        gu()
    evg = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in evg:
        flush.zero_()
        a.record(stream)
        gu()
        b.record(stream)
    torch.cuda.synchronize()
    gu_ms = statistics.median([a.elapsed_time(b) for a, b in evg])
    st = sq.get_last_error()
    if st != sq.OK:
        raise RuntimeError(sq.status_name(st))
    lin = {"gate": (inter, hidden), "up": (inter, hidden), "down": (hidden, inter)}
    flops = {k: 2.0 * rows * no * kk * (1.0 + n / m) for k, (no, kk) in lin.items()}
    counts = np.diff(offsets)
    padded = int(128 * ((counts + 127) // 128).sum())
    gemm_ms = sum(per[k] for k in lin)
    peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    achieved = sum(flops.values()) / (gemm_ms / 1e3) / 1e12
    return {"case": f"moe:{tokens}", "workload": "Qwen3-30B-A3B MoE FFN: hidden 2048, 128 experts x "
            "intermediate 768, top-8 of N(0,1) gate logits; gate/up/down grouped SharQ linears, NVFP4 2:4",
            "tokens": tokens, "rows": rows, "padded_rows": padded, "ms_per_step": step_ms,
            "tokens_per_s": tokens / (step_ms / 1e3), "ms": per,
            "gemm_roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                              "frac": achieved / peak, "flops_algorithmic": sum(flops.values()),
                              "peak_source": peak_src + " (bf16 burst x 4)"},
            "fused_gate_up": {"ms": gu_ms, "separate_ms": per["gate"] + per["up"],
                              "frac": (flops["gate"] + flops["up"]) / (gu_ms / 1e3) / 1e12 / peak,
                              "step_ms_with_fused": step_ms - per["gate"] - per["up"] + gu_ms},
            "gpu_launches_per_step": launches, "steps": args.steps,
            "warmup": args.warmup, "l2": "flushed (256 MB write) before every step"}


def main():
    args = parse_args()
    world, rank, local = dist_setup(args)
    try:
        if args.case:
            res = run_case(args, world, rank, local)
        elif args.impl == "reference":
            res = run_reference(args, world, rank)
        else:
            res = run_sharq(args, world, rank, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    main()
