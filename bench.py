#!/usr/bin/env python3
"""Benchmark of the shifted-window attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--only] [--impl native|reference]

A step is one call of swin_window_attn_fwd (the whole hot path: CPB
evaluation where the workload has one, then the attention kernel) over one
batch of the workload, inputs resident in HBM.  L2 is flushed (a 256 MB
write) before every timed step; each step is timed with CUDA events on the
library's stream and the median step is reported.  For N > 1 (torchrun)
every rank runs its own batch (weak scaling, no collective on the data path)
and the time is the max over ranks.

Prints one JSON line.  The headline workload (FlashSwin-T dense tokens, M=32,
unless --workload) gives ``value`` (whole-job tokens/s), ``tflops``,
``roofline`` (the attention kernel against the measured bf16 peak, DRAM
traffic from the committed ncu summary of the same kernel source, and
``exp_bound``: the share of the all-MUFU exponential bound it reaches) and
``e2e`` (host buffers, every step's copies in the timed region: the H2D copy
of q, k, v from pinned host memory and the D2H copy of the output, on their
own streams with two device buffer sets, so one step's copies overlap its
neighbours' copies and kernels; steady-state time per step over the loop;
``e2e.serial_ms_per_step`` is the same step with copies and call in one
stream).  ``workloads`` repeats
those figures for every bf16 workload (headline first; --only skips the
others), with the CPB kernel's time in both forms where a workload has one;
every bf16, d = 32 workload runs on a tensor-core kernel (the TMA kernel, or
the rectangle kernel for interleaved and small windows) and is set against
the bf16 peak; one that ran on the CUDA cores would be set against their fp32
peak ("bound": "alu").
``backward`` times swin_window_attn_bwd on the same workloads (--no-backward
skips it); ``block`` times the attention half of a Swin V2 block
(swin_attn_block_fwd) and its projection steps against HBM (--no-block).
Also: SM clocks sampled during the timed loops, the number of this library's
kernel launches timed, and ``cpu_baseline`` (the oracle on the host cores and
on one core).  ``--impl reference`` times the CPU oracle (the project's plain
double-precision statement of the method) on the host cores on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from vision_transformer_shifted_window_b200 import synthetic as syn  # noqa: E402

METRIC = "window-attn fwd tokens/s and TFLOP/s (bf16, 1 B200) as % of tensor roofline"
DEFAULT_WORKLOAD = 3  # FlashSwin dense tokens, M=32: the tensor-bound workload
L2_FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------------------
# algorithmic work per workload
# ---------------------------------------------------------------------------
def _seg_lengths(L, M, s):
    if s == 0:
        starts = list(range(0, L, M))
    else:
        starts = [0] + list(range(s, L, M))
    ends = starts[1:] + [L]
    return [b - a for a, b in zip(starts, ends) if b > a]


def _window_counts(L, M, s):
    """Real tokens per rolled-frame window along one axis (Swin's count)."""
    Lp = -(-L // M) * M
    out = []
    for w in range(Lp // M):
        out.append(sum(1 for u in range(w * M, w * M + M) if (u + s) % Lp < L))
    return out


def _interleaved_lengths(L, M):
    """Tokens per interleaved window along one axis: G = ceil(L/M) windows,
    window a holds a + G i inside the axis."""
    G = -(-L // M)
    return [-(-(L - a) // G) for a in range(G)]


def work(w: syn.Workload, B=None):
    B = w.B if B is None else B
    s = w.shifts[0]
    if w.partition == 1:  # interleaved windows: no padding, no mask
        win = exact = (sum(n * n for n in _interleaved_lengths(w.H, w.M)) *
                       sum(n * n for n in _interleaved_lengths(w.W, w.M)))
    else:
        win = sum(n * n for n in _window_counts(w.H, w.M, s)) * sum(n * n for n in _window_counts(w.W, w.M, s))
        exact = sum(n * n for n in _seg_lengths(w.H, w.M, s)) * sum(n * n for n in _seg_lengths(w.W, w.M, s))
    C = w.heads * w.d
    esz = 4 if w.dtype == "f32" else 2
    return {
        "tokens": B * w.H * w.W,
        "flops_std": 4.0 * w.d * w.heads * B * win,      # masked pairs in a window included
        "flops_exact": 4.0 * w.d * w.heads * B * exact,  # only pairs that enter a softmax
        "exps": float(w.heads * B * exact),
        "bytes": float(4 * esz * C * B * w.H * w.W),     # Q, K, V read once, O written once
    }


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def read_traffic(kernel: str, workload: syn.Workload):
    """dram read+write bytes per launch from a committed ncu summary, if the
    summary was taken on the current kernel source (else None)."""
    fn = os.path.join(ROOT, "profiles", "%s_%s.txt" % (kernel, workload.name))
    if not os.path.exists(fn):
        return None
    kv = {}
    for line in open(fn):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    src = os.path.join(ROOT, "vision_transformer_shifted_window_b200", "csrc", kv.get("source_file", ""))
    if not os.path.isfile(src) or "source_sha1" not in kv or "dram_bytes_per_launch" not in kv:
        return None
    if hashlib.sha1(open(src, "rb").read()).hexdigest() != kv["source_sha1"]:
        return None
    return float(kv["dram_bytes_per_launch"])


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", "swin_clocks_%d_%d.csv" % (os.getpid(), gpu_index))

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons, n = [], None, set(), 0
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            n += 1
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": n}


# ---------------------------------------------------------------------------
# native arm
# ---------------------------------------------------------------------------
def make_device_inputs(w: syn.Workload, device, rank: int):
    import torch
    inp = syn.make_inputs(w, seed=1000 + w.index + 7919 * rank)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    q, k, v = (dev(inp[n]).to(dt) for n in ("q", "k", "v"))
    kw = {}
    if "tau" in inp:
        kw["tau"] = dev(inp["tau"])
    if "table" in inp:
        kw["bias_table"] = dev(inp["table"])
    if "w1" in inp:
        kw["cpb"] = tuple(dev(inp[n]) for n in ("w1", "b1", "w2", "b2"))
    if "rope_freqs" in inp:
        kw["rope_freqs"] = dev(inp["rope_freqs"])
    return q, k, v, kw


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


MUFU_EX2_PER_CLK_PER_SM = 16  # B200: exp2 throughput of the special-function unit


def exp_bound(wk: dict, sms: int, clock_mhz: float, kernel_ms: float) -> dict:
    """Time the exponentials alone need if every one ran on the MUFU (one per
    attended pair), and the fraction of it the kernel achieves: at d = 32 this,
    not the tensor pipe, is the ceiling of an all-MUFU softmax."""
    t_ms = wk["exps"] / (MUFU_EX2_PER_CLK_PER_SM * sms * clock_mhz * 1e6) * 1e3
    return {"ex2_per_clk_per_sm": MUFU_EX2_PER_CLK_PER_SM, "sms": sms, "clock_mhz": clock_mhz,
            "bound_ms": round(t_ms, 5), "frac": round(t_ms / kernel_ms, 4)}


def whole_job(wk: dict, world: int, ms_max: float) -> dict:
    """Whole-job rates of `world` replica ranks that each processed one
    workload `wk` (weak scaling), timed as the slowest rank's ms per step."""
    sec = ms_max * 1e-3
    return {"tokens_per_s": wk["tokens"] * world / sec,
            "tflops": wk["flops_std"] * world / sec / 1e12,
            "tflops_exact": wk["flops_exact"] * world / sec / 1e12}


FP32_LANES_PER_SM = 128  # B200: fp32 FMA lanes per SM per clock


def fwd_kernel(w: syn.Workload) -> str:
    """The kernel the library runs this workload's forward on: the rectangle
    tensor-core kernel (bf16, d = 32, M <= 32, interleaved windows or M <= 8),
    the TMA tensor-core kernel (other bf16, d = 32 shifted windows, no bias
    table above M = 32) or the CUDA cores."""
    has_table = w.mode != 2 and w.bias
    if w.dtype == "bf16" and w.d == 32 and w.M <= 32 and (w.partition == 1 or w.M <= 8):
        return "fwd_tc_rect"
    if w.dtype == "bf16" and w.d == 32 and w.partition == 0 and (not has_table or w.M <= 32):
        return "attn_tc"
    return "attn_simt"


def on_tensor_cores(w: syn.Workload) -> bool:
    return fwd_kernel(w) != "attn_simt"


def alu_peak_tflops(sms: int, clock_mhz: float) -> float:
    """fp32 FMA peak of the CUDA cores: SMs x 128 lanes x 2 flop x SM clock."""
    return sms * FP32_LANES_PER_SM * 2 * clock_mhz * 1e6 / 1e12


def config_of(w: syn.Workload, world: int) -> dict:
    """The workload as both arms name it (same keys and values)."""
    return {"workload": w.name, "B": w.B, "H": w.H, "W": w.W, "heads": w.heads, "d": w.d, "M": w.M,
            "shift": w.shifts[0], "mode": ["dot+bias", "cosine+cpb", "rope"][w.mode],
            "partition": ["shifted", "interleaved"][w.partition],
            "global_batch": w.B * world, "parallelism": "replicas x%d" % world,
            "l2": "flushed before every timed step (256 MB write)", "timing": "median of per-step CUDA events"}


def _median(xs):
    return float(np.median(np.asarray(xs, dtype=np.float64)))


class Timer:
    """Per-step CUDA-event timing on the library's stream, with an L2 flush
    (a write larger than L2) before every timed step."""

    def __init__(self, device, stream):
        import torch
        self.torch, self.device, self.stream = torch, device, stream
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def loop(self, fn, n, flush_l2=True):
        torch = self.torch
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        with torch.cuda.stream(self.stream):
            for i in range(n):
                if flush_l2:
                    self.flush.fill_(i & 0xFF)
                evs[i][0].record(self.stream)
                fn()
                evs[i][1].record(self.stream)
        torch.cuda.synchronize(self.device)
        return [a.elapsed_time(b) for a, b in evs]


def time_workload(w: syn.Workload, args, timer, rank: int, world: int, peaks: dict, sms: int, clock_mhz: float,
                  with_e2e: bool):
    """One workload: the whole call (CPB + attention) per step, the attention
    kernel alone, and, for the headline, the end-to-end call through host
    buffers.  Returns (entry, launches of this library's kernels timed)."""
    import torch
    from vision_transformer_shifted_window_b200 import swin_attn as sa
    device, stream = timer.device, timer.stream
    s = w.shifts[0]
    q, k, v, kw = make_device_inputs(w, device, rank)
    out = torch.empty_like(q)
    ws_bytes = sa.swin_window_attn_workspace_size(w.M, w.heads, w.mode, "bias_table" in kw)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=device)
    launches_per_step = 2 if "cpb" in kw else 1

    def step():
        sa.swin_window_attn_fwd(q, k, v, w.M, s, w.mode, out=out, workspace=ws, stream=stream,
                                partition=w.partition, **kw)

    timer.loop(step, max(args.warmup, 3))
    if sa.swin_stream_status(stream) != 0:
        raise RuntimeError("device status after warm-up of %s" % w.name)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    times = timer.loop(step, args.steps)
    launches = launches_per_step * args.steps
    ms = max_over_ranks(_median(times), world, device)
    wk = work(w)
    job = whole_job(wk, world, ms)

    # the attention kernel alone (the bias table given, no CPB evaluation)
    cpb_us = None
    if "cpb" in kw:
        table = sa.swin_cpb_eval(w.M, w.heads, *kw["cpb"], stream=stream)
        kw_k = {kk: vv for kk, vv in kw.items() if kk != "cpb"}
        kw_k["bias_table"] = table

        def kstep():
            sa.swin_window_attn_fwd(q, k, v, w.M, s, w.mode, out=out, stream=stream, partition=w.partition,
                                    **kw_k)
        timer.loop(kstep, 3)
        ktimes = timer.loop(kstep, args.steps)
        launches += args.steps
        cpb_us = {}
        for name, form in (("paper", sa.SWIN_CPB_PAPER), ("code", sa.SWIN_CPB_CODE)):
            def cstep(form=form):
                sa.swin_cpb_eval_form(w.M, w.heads, *kw["cpb"], form, 0, out=table, stream=stream)
            timer.loop(cstep, 3, flush_l2=False)
            ct = timer.loop(cstep, 20, flush_l2=False)
            launches += 20
            cpb_us[name] = round(1e3 * _median(ct), 2)
    else:
        ktimes = times
    k_ms = max_over_ranks(_median(ktimes), world, device)
    achieved = wk["flops_std"] / (k_ms * 1e-3) / 1e12
    hbm = wk["bytes"] / (k_ms * 1e-3) / 1e9
    kname = fwd_kernel(w)
    if on_tensor_cores(w):
        peak, bound, src = peaks["bf16_tflops"], "tensor", peaks["source"] + " (burst)"
    else:  # the CUDA-core kernel: fp32 FMA lanes
        peak, bound = alu_peak_tflops(sms, clock_mhz), "alu"
        src = "derived: %d SMs x %d fp32 lanes x 2 flop x %.0f MHz" % (sms, FP32_LANES_PER_SM, clock_mhz)
    roofline = {"bound": bound, "achieved": round(achieved, 2), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "traffic": read_traffic(kname, w),
                "peak_source": src, "kernel": kname,
                "kernel_ms": round(k_ms, 5), "algorithmic_bytes": wk["bytes"],
                "hbm_achieved_gbs": round(hbm, 1), "hbm_frac": round(hbm / peaks["hbm_gbs"], 4),
                "attainable_frac": round(achieved / min(peak, peaks["hbm_gbs"] * wk["flops_std"] / wk["bytes"] / 1e3),
                                         4),
                "exp_bound": exp_bound(wk, sms, clock_mhz, k_ms)}
    entry = {"workload": w.name, "config": {"B": w.B, "H": w.H, "W": w.W, "heads": w.heads, "d": w.d, "M": w.M,
                                            "shift": s, "mode": ["dot+bias", "cosine+cpb", "rope"][w.mode],
                                            "partition": ["shifted", "interleaved"][w.partition]},
             "ms_per_step": round(ms, 5), "tokens_per_s": round(job["tokens_per_s"], 1),
             "tflops": round(job["tflops"], 2), "tflops_exact_pairs": round(job["tflops_exact"], 2),
             "roofline": roofline}
    if cpb_us:
        entry["cpb_us"] = cpb_us
    if with_e2e:
        # end to end through host buffers: H2D of q/k/v, the call, D2H of out
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            step()
            hout.copy_(out, non_blocking=True)
        timer.loop(e2e_step, 3, flush_l2=False)
        n_e2e = max(3, min(args.steps, 20))
        etimes = timer.loop(e2e_step, n_e2e, flush_l2=False)
        launches += launches_per_step * n_e2e
        serial_ms = max_over_ranks(_median(etimes), world, device)
        # pipelined: step i copies into buffer set i % 2 on the H2D stream,
        # computes on the library's stream, copies back on the D2H stream;
        # events order every reuse of a buffer set after its previous step
        sets = [(q, k, v, out, ws)] + [tuple(torch.empty_like(t) for t in (q, k, v, out)) + (torch.empty_like(ws),)]
        h2d, d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev = lambda: torch.cuda.Event()
        in_ready, computed, out_read = [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def pipelined(n):
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            h2d.wait_event(t0)
            d2h.wait_event(t0)
            for i in range(n):
                j = i & 1
                qq, kk, vv, oo, ww = sets[j]
                if i >= 2:
                    h2d.wait_event(computed[j])  # the call of step i - 2 has read this set
                with torch.cuda.stream(h2d):
                    qq.copy_(hq, non_blocking=True)
                    kk.copy_(hk, non_blocking=True)
                    vv.copy_(hv, non_blocking=True)
                    in_ready[j].record(h2d)
                stream.wait_event(in_ready[j])
                if i >= 2:
                    stream.wait_event(out_read[j])  # the D2H of step i - 2 has read this output
                sa.swin_window_attn_fwd(qq, kk, vv, w.M, s, w.mode, out=oo, workspace=ww, stream=stream,
                                        partition=w.partition, **kw)
                computed[j].record(stream)
                d2h.wait_event(computed[j])
                with torch.cuda.stream(d2h):
                    hout.copy_(oo, non_blocking=True)
                    out_read[j].record(d2h)
            stream.wait_event(out_read[(n - 1) & 1])
            stream.wait_event(in_ready[(n - 1) & 1])
            t1.record(stream)
            torch.cuda.synchronize(device)
            return t0.elapsed_time(t1) / n
        pipelined(3)
        e_ms = max_over_ranks(pipelined(n_e2e), world, device)
        launches += launches_per_step * n_e2e
        entry["e2e"] = {"value": round(wk["tokens"] * world / (e_ms * 1e-3), 1), "unit": "tokens/s",
                        "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
                        "d2h_bytes_per_step": out.numel() * out.element_size(), "ms_per_step": round(e_ms, 4),
                        "serial_ms_per_step": round(serial_ms, 4)}
    if sa.swin_stream_status(stream) != 0:
        raise RuntimeError("device status after the timed loops of %s" % w.name)
    del q, k, v, out, ws
    torch.cuda.empty_cache()
    return entry, launches


def bwd_on_tensor_cores(w: syn.Workload) -> bool:
    """Whether the library runs this workload's backward on the tensor cores
    (bf16, d = 32, M <= 32, either partition)."""
    return w.dtype == "bf16" and w.d == 32 and w.M <= 32


def time_backward(w: syn.Workload, args, timer, rank: int, world: int, sms: int, clock_mhz: float, peaks: dict):
    """The backward pass (swin_window_attn_bwd: dq, dk, dv and the parameter
    gradients, softmax recomputed) of one workload, bf16 gradients.  Its
    algorithmic work is five products of 2 d flops per attended pair (S, dP,
    dV, dK, dQ), measured against the bf16 tensor peak where the tensor-core
    kernels run (else the CUDA cores' fp32 FMA peak); its exponentials, three
    per pair (the statistics pass and both gradient passes), give the MUFU
    bound beside it.  Returns (entry, launches)."""
    import torch
    from vision_transformer_shifted_window_b200 import swin_attn as sa
    device, stream = timer.device, timer.stream
    s = w.shifts[0]
    q, k, v, kw = make_device_inputs(w, device, rank)
    g = torch.from_numpy(syn.make_dout(w, seed=5000 + w.index + 7919 * rank)).to(device).to(q.dtype)
    if "cpb" in kw:
        kw["bias_table"] = sa.swin_cpb_eval(w.M, w.heads, *kw.pop("cpb"), stream=stream)
    ws = torch.empty(sa.swin_window_attn_bwd_workspace_size(*q.shape, w.M), dtype=torch.uint8, device=device)
    params = ("bias_table" in kw) or w.mode != 0

    def step():
        sa.swin_window_attn_bwd(q, k, v, g, w.M, s, w.mode, workspace=ws, stream=stream, partition=w.partition,
                                **kw)
    n = max(3, min(args.steps, 10))
    timer.loop(step, 2)
    times = timer.loop(step, n)
    if sa.swin_stream_status(stream) != 0:
        raise RuntimeError("device status after the backward of %s" % w.name)
    ms = max_over_ranks(_median(times), world, device)
    wk = work(w)
    flops = 2.5 * wk["flops_exact"]
    achieved = flops / (ms * 1e-3) / 1e12
    tc = bwd_on_tensor_cores(w)
    if tc:
        peak, bound, kname, src = peaks["bf16_tflops"], "tensor", "bwd_tc_q + bwd_tc_kv", peaks["source"] + " (burst)"
    else:
        peak, bound, kname = alu_peak_tflops(sms, clock_mhz), "alu", "bwd_q + bwd_kv (CUDA cores)"
        src = "derived: %d SMs x %d fp32 lanes x 2 flop x %.0f MHz" % (sms, FP32_LANES_PER_SM, clock_mhz)
    exps = dict(wk, exps=3 * wk["exps"])
    entry = {"workload": w.name, "ms_per_step": round(ms, 4),
             "tokens_per_s": round(wk["tokens"] * world / (ms * 1e-3), 1),
             "roofline": {"bound": bound, "achieved": round(achieved, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
                          "frac": round(achieved / peak, 4),
                          "traffic": read_traffic("attn_bwd_tc", w) if tc else None, "kernel": kname,
                          "algorithmic_flops": flops, "peak_source": src, "kernel_ms": round(ms, 5),
                          "exp_bound": exp_bound(exps, sms, clock_mhz, ms)}}
    del q, k, v, g, ws
    torch.cuda.empty_cache()
    return entry, n * ((3 if params else 2))


def time_block(w: syn.Workload, args, timer, rank: int, world: int, peaks: dict):
    """The attention half of a Swin V2 block on one workload (swin_attn_block_fwd:
    qkv projection, the attention, output projection with the residual
    post-norm), bf16, and its two projection steps alone.  The projections
    are memory-bound at these widths (K = C <= 512), so each step is set
    against HBM: its algorithmic bytes are the tensors it must read and write
    once (x and W in, q, k, v out; a, x and W_o in, out out).  Returns
    (entry, launches)."""
    import torch
    from vision_transformer_shifted_window_b200 import swin_attn as sa
    device, stream = timer.device, timer.stream
    s = w.shifts[0]
    _, _, _, kw = make_device_inputs(w, device, rank)
    p = syn.make_block_inputs(w, seed=9000 + w.index + 7919 * rank)
    dev = lambda a, dt=None: torch.from_numpy(np.ascontiguousarray(a)).to(device).to(dt or torch.float32)
    bf = torch.bfloat16
    x, wq, wo = dev(p["x"], bf), dev(p["w_qkv"], bf), dev(p["w_o"], bf)
    bq, bo, ga, be = (dev(p[n]) for n in ("b_qkv", "b_o", "gamma", "beta"))
    B, H, W, C = x.shape
    tokens = B * H * W
    out = torch.empty_like(x)
    ws = torch.empty(sa.swin_attn_block_workspace_size(B, H, W, w.heads, w.d, w.M, w.mode, "bias_table" in kw, bf),
                     dtype=torch.uint8, device=device)
    q, k, v, a = (torch.empty_like(x) for _ in range(4))
    wsq = torch.empty(max(sa.lib().swin_qkv_proj_workspace_size(tokens, C), 256), dtype=torch.uint8, device=device)
    wsp = torch.empty(max(sa.lib().swin_proj_postnorm_workspace_size(tokens, C), 256), dtype=torch.uint8,
                      device=device)
    n = max(3, min(args.steps, 20))

    def block():
        sa.swin_attn_block_fwd(x, w.heads, wq, bq, wo, bo, ga, be, w.M, s, w.mode, out=out, workspace=ws,
                               stream=stream, partition=w.partition, **kw)

    def qkv():
        sa.swin_qkv_proj(x, wq, bq, workspace=wsq, stream=stream)

    def post():
        sa.swin_proj_postnorm_residual(a, wo, bo, x, ga, be, out=out, workspace=wsp, stream=stream)
    res = {}
    for name, fn in (("block", block), ("qkv_proj", qkv), ("proj_postnorm", post)):
        timer.loop(fn, 2)
        res[name] = max_over_ranks(_median(timer.loop(fn, n)), world, device)
    if sa.swin_stream_status(stream) != 0:
        raise RuntimeError("device status after the block of %s" % w.name)
    e = 2  # bf16 bytes
    bytes_qkv = tokens * C * e * 4 + 3 * C * C * e
    bytes_post = tokens * C * e * 3 + C * C * e
    hbm = peaks["hbm_gbs"]
    gbs = lambda b, ms: b / (ms * 1e-3) / 1e9
    entry = {"workload": w.name, "block_ms": round(res["block"], 4),
             "block_tokens_per_s": round(tokens * world / (res["block"] * 1e-3), 1),
             "qkv_proj": {"ms": round(res["qkv_proj"], 4), "algorithmic_bytes": bytes_qkv,
                          "achieved_gbs": round(gbs(bytes_qkv, res["qkv_proj"]), 1),
                          "frac_hbm": round(gbs(bytes_qkv, res["qkv_proj"]) / hbm, 4)},
             "proj_postnorm": {"ms": round(res["proj_postnorm"], 4), "algorithmic_bytes": bytes_post,
                               "achieved_gbs": round(gbs(bytes_post, res["proj_postnorm"]), 1),
                               "frac_hbm": round(gbs(bytes_post, res["proj_postnorm"]) / hbm, 4)},
             "peak": {"hbm_gbs": hbm, "source": peaks["source"]}}
    # this library's kernels per timed call (the cuBLASLt GEMMs are not counted):
    # block = split, [CPB,] attention, post-norm; each projection step = 1
    mine_block = 3 + (1 if "cpb" in kw else 0)
    del x, out, ws, q, k, v, a, wsq, wsp
    torch.cuda.empty_cache()
    return entry, n * (mine_block + 1 + 1)


def run_native(args, rank: int, world: int, local_rank: int):
    import torch
    from vision_transformer_shifted_window_b200 import build as swin_build

    swin_build.build()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device)
    timer = Timer(device, stream)
    peaks = read_peaks()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    headline = syn.WORKLOADS[args.workload]
    others = [] if args.only else [i for i in sorted(syn.WORKLOADS)
                                   if i != args.workload and syn.WORKLOADS[i].dtype == "bf16"]
    sampler = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                           else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank]))
    sampler.start()
    # clocks are sampled over the timed loops; the exponential bound uses the
    # SM clock the box advertises (the sampled median is reported beside it)
    clock_guess = 1965.0
    entry, launches = time_workload(headline, args, timer, rank, world, peaks, sms, clock_guess, with_e2e=True)
    other_entries = []
    for idx in (others if args.part in ("all", "fwd") else []):
        e, n = time_workload(syn.WORKLOADS[idx], args, timer, rank, world, peaks, sms, clock_guess, False)
        other_entries.append(e)
        launches += n
    block_entries = []
    if not args.no_block and args.part in ("all", "block"):
        for idx in [args.workload] + others:
            e, n = time_block(syn.WORKLOADS[idx], args, timer, rank, world, peaks)
            block_entries.append(e)
            launches += n
    bwd_entries = []
    if not args.no_backward and args.part in ("all", "bwd"):
        for idx in [args.workload] + others:
            e, n = time_backward(syn.WORKLOADS[idx], args, timer, rank, world, sms, clock_guess, peaks)
            bwd_entries.append(e)
            launches += n
    clocks = sampler.stop()
    sm_mhz = float(clocks["sm_mhz"] or clocks["sm_max_mhz"] or clock_guess)
    wk = work(headline)
    for e, w in [(entry, headline)] + [(o, syn.WORKLOADS[i]) for o, i in zip(other_entries, others)]:
        e["roofline"]["exp_bound"] = exp_bound(work(w), sms, sm_mhz, e["roofline"]["kernel_ms"])
        if e["roofline"]["bound"] == "alu":  # the derived peak at the sampled clock
            pk = alu_peak_tflops(sms, sm_mhz)
            e["roofline"].update(peak=round(pk, 1), frac=round(e["roofline"]["achieved"] / pk, 4),
                                 peak_source="derived: %d SMs x %d fp32 lanes x 2 flop x %.0f MHz (sampled)"
                                             % (sms, FP32_LANES_PER_SM, sm_mhz))
    for e, i in zip(bwd_entries, [args.workload] + others):
        w = syn.WORKLOADS[i]
        e["roofline"]["exp_bound"] = exp_bound(dict(work(w), exps=3 * work(w)["exps"]), sms, sm_mhz,
                                               e["roofline"]["kernel_ms"])
        if e["roofline"]["bound"] == "alu":
            pk = alu_peak_tflops(sms, sm_mhz)
            e["roofline"].update(peak=round(pk, 1), frac=round(e["roofline"]["achieved"] / pk, 4),
                                 peak_source="derived: %d SMs x %d fp32 lanes x 2 flop x %.0f MHz (sampled)"
                                             % (sms, FP32_LANES_PER_SM, sm_mhz))
    line = {
        "metric": METRIC, "value": entry["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": entry["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if headline.dtype == "bf16" else "f32", "data": "synthetic",
        "config": config_of(headline, world),
        "tflops": entry["tflops"], "tflops_exact_pairs": entry["tflops_exact_pairs"],
        "roofline": entry["roofline"],
        "e2e": entry["e2e"],
        "clocks": clocks, "gpu_launches": launches,
        "workloads": [{k: v for k, v in entry.items() if k != "e2e"}] + other_entries,
        "backward": bwd_entries,
        "block": block_entries,
    }
    return line, headline


def cpu_model() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.lower().startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def run_cpu_baseline(w: syn.Workload, budget_s: float):
    """Time the oracle on a bounded, seeded sample of the workload's queries
    (drawn without replacement from every image of the batch), on all host
    cores and on one core."""
    import oracle
    inp = syn.make_inputs(w)
    s = w.shifts[0]
    table = None
    if "table" in inp:
        table = inp["table"]
    elif "w1" in inp:
        table = oracle.cpb_table(w.M, w.heads, inp["w1"], inp["b1"], inp["w2"], inp["b2"])
    rng = np.random.default_rng(99)
    n_all = w.B * w.H * w.W

    def run(nq, nthreads=0):
        ids = np.sort(rng.choice(n_all, size=min(nq, n_all), replace=False))
        t0 = time.perf_counter()
        oracle.window_attn(inp["q"], inp["k"], inp["v"], w.M, s, w.mode, tau=inp.get("tau"), table=table,
                           rope_freqs=inp.get("rope_freqs"), queries=ids, nthreads=nthreads,
                           partition=w.partition)
        return len(ids), time.perf_counter() - t0

    def sized(budget, nthreads):
        nq, t = run(64, nthreads)
        while t < 0.3 and nq < n_all:
            nq, t = run(nq * 4, nthreads)
        return run(int(min(n_all, max(nq, nq * budget / max(t, 1e-6)))), nthreads)

    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    nq, t = sized(budget_s, cores)
    nq1, t1 = sized(max(1.0, budget_s / 4), 1)
    return {"value": round(nq / t, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "single_core_tokens_per_s": round(nq1 / t1, 2),
            "sample": "%d query tokens drawn without replacement from all %d images of %s (all %d heads), %.1f s "
                      "on %d threads; %d tokens on 1 thread, %.1f s" % (nq, w.B, w.name, w.heads, t,
                                                                       cores, nq1, t1),
            "seconds": round(t, 2)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD, choices=sorted(syn.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=("native", "reference"))
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work to time")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", action="store_true", help="time the headline workload alone")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward-pass measurements")
    ap.add_argument("--no-block", action="store_true", help="skip the block (projections + post-norm) measurements")
    ap.add_argument("--part", default="all", choices=("all", "fwd", "bwd", "block"),
                    help="time one part only (for profiling captures): the forward lines, the backward or the block "
                         "(the JSON line then carries the forward headline plus that part)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = syn.WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return 0
        budget = max(1.0, min(60.0, args.cpu_budget * max(1, args.steps) / 10.0))
        cb = run_cpu_baseline(w, budget)
        line = {"metric": METRIC, "impl": "reference", "value": cb["value"], "unit": "tokens/s", "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": config_of(w, world),
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    line, w = run_native(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = run_cpu_baseline(w, args.cpu_budget)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
