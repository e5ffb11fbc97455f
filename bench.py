#!/usr/bin/env python
"""Benchmark of the UNet attention hot path on B200.

One step = the attention set of one 512x512 Stable Diffusion 1.4 UNet step:
16 transformer blocks, each a self-attention (M = N = h*w) and a
cross-attention (M = 77), B = 2 (classifier-free guidance pair), H = 8,
d = 40 / 80 / 160, fp16 inputs.  Each call runs the form the paper's policy
picks ("Speed Is All You Need", news summary, FlashAttention paragraph: the
FlashAttention kernel for d = 40, the partially fused softmax elsewhere), so a
step exercises every kernel: flash, qk_stats and softmax_av.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints ONE JSON line (rank 0).  `value` is whole-job TFLOP/s (algorithmic
FLOPs 4*B*H*N*M*d summed over the set and over ranks, divided by the max-over-
ranks device time of K steps).  Steps replay a CUDA graph of the set; two
independent input sets (each larger than the 126 MB L2) alternate, so no step
finds its inputs in L2.  Multi-GPU runs are independent replicas (the work
needs no exchange); NCCL carries only the barrier and the max of the timings.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

# Sources each profiled kernel is built from; a committed ncu summary
# (profiles/<name>.json) counts only while its recorded digest matches them.
CSRC = "diffusion_unet_attention_b200/csrc/"
KERNEL_SRC = {
    "flash": (CSRC + "flash.cuh", CSRC + "sm100.cuh", CSRC + "sdattn.cu"),
    "qk_stats": (CSRC + "qk_stats.cuh", CSRC + "sm100.cuh", CSRC + "sdattn.cu"),
    "softmax_av": (CSRC + "softmax_av.cuh", CSRC + "sm100.cuh", CSRC + "sdattn.cu"),
}
PROFILE_JSON = {k: os.path.join(ROOT, "profiles", f"{k}_64x64_self_d40.json") for k in KERNEL_SRC}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["sdattn", "reference"], default="sdattn")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-side", action="store_true",
                    help="time the step set only (no per-form, per-kernel or end-to-end extras)")
    ap.add_argument("--case", default=None,
                    help="FORM:WORKLOAD, e.g. flash:self64 -- run one form (flash, qk_stats, softmax_av, "
                         "qk_stats_f16a, softmax_av_f16a, partial, f16a, three_pass, or all three kernels) on one workload; or conv3x3:CxH, e.g. conv3x3:320x64 -- one "
                         "Winograd 3x3 convolution (batch 2, C = K) (for profilers)")
    ap.add_argument("--reps", type=int, default=3)
    return ap.parse_args()


# ----------------------------------------------------------------------------
# workload
# ----------------------------------------------------------------------------
CALLS = synth.unet_step_set()
STEP_FLOPS = sum(c.flops for c in CALLS)
WORKLOAD = ("SD1.4 512x512 UNet step attention set: 16 transformer blocks x (self M=N=hw, cross M=77), "
            "B=2, H=8, d=40/80/160, fp16 N(0,1); flash for d=40, partially fused softmax otherwise")


# bytes of one input set (Q, K, V of every call, fp16)
SET_BYTES = sum(2 * c.B * c.H * (c.N + 2 * c.M) * c.d for c in CALLS)


def job_config(world: int) -> dict:
    """The `config` of the JSON line, the same for both arms."""
    return {"workload": WORKLOAD, "calls_per_step": len(CALLS), "flops_per_step": STEP_FLOPS,
            "accumulate": "f32", "l2": "two input sets of %.0f MB alternate (each > 126 MB L2)" % (SET_BYTES / 1e6),
            "timing": "CUDA graph replay per step, CUDA events", "parallelism": f"replicas x{world}"}


def policy_form(call) -> str:
    return "flash" if call.d == 40 else "partial"


def is_dominant(call) -> bool:
    return call.d == 40 and call.N == 4096 and call.M == 4096


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def source_digest(kernel: str = "flash") -> str:
    """First 16 hex digits of the SHA-256 over the kernel's source files."""
    h = hashlib.sha256()
    for rel in KERNEL_SRC[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled(kernel: str = "flash"):
    """The committed ncu figures of `kernel` on the 64x64 self-attention
    (profiles/<kernel>_64x64_self_d40.json), or None when they are missing or
    were taken on other sources than the current ones."""
    try:
        with open(PROFILE_JSON[kernel]) as f:
            prof = json.load(f)
    except (OSError, ValueError):
        return None
    if prof.get("source_digest") != source_digest(kernel):
        return None
    return prof


def profiled_traffic(kernel: str = "flash"):
    """Per-launch DRAM bytes (read + write) of `kernel` from its current profile."""
    prof = profiled(kernel)
    if prof is None:
        return None
    return float(prof["dram_bytes_read"] + prof["dram_bytes_write"])


# ----------------------------------------------------------------------------
# ranks: independent replicas; only the timing crosses processes
# ----------------------------------------------------------------------------
def max_over_ranks(value: float, dist, device) -> float:
    """The largest `value` of all ranks (the job's time is its slowest rank's)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flops_per_step: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs the full step set (weak scaling)."""
    return world * flops_per_step * steps / (elapsed_ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, smax, power, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_median": statistics.median(power) if power else None}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------
class StepSet:
    """Device-resident inputs, outputs and scratch for one step set."""

    def __init__(self, sd, torch, device, set_id: int):
        self.sd, self.torch, self.device = sd, torch, device
        self.inputs = []
        self.device = device
        for ci, call in enumerate(CALLS):
            q, k, v = synth.make_qkv(call, synth.STEP_SET_ID + 10 * set_id, call_id=ci)
            tq, tk, tv = (torch.from_numpy(x).to(device) for x in (q, k, v))
            o = torch.empty_like(tq)
            self.inputs.append((call, tq, tk, tv, o))

    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for _, q, k, v, _ in self.inputs for t in (q, k, v))

    def d2h_bytes(self):
        return sum(o.numel() * o.element_size() for *_, o in self.inputs)


class Scratch:
    """A, LS and workspace shared by every call of a stream."""

    def __init__(self, sd, torch, device, calls):
        self.sd, self.torch = sd, torch
        a_elems = max(c.B * c.H * c.N * ((c.M + 3) // 4 * 4) for c in calls)
        ls_elems = max(c.B * c.H * c.N * 2 for c in calls)
        self.a = torch.empty(a_elems, dtype=torch.float32, device=device)
        self.ls = torch.empty(ls_elems, dtype=torch.float32, device=device)
        ws = max(sd.workspace_bytes(sd.make_desc(c.B, c.H, c.N, c.M, c.d, torch.float16, 1.0)) for c in calls)
        self.ws = torch.zeros(max(ws, 256), dtype=torch.uint8, device=device)

    def views(self, call):
        """A [B,H,N,lda] and LS [B,H,N,2] views of the shared scratch for `call`."""
        lda = (call.M + 3) // 4 * 4
        a = self.a[:call.B * call.H * call.N * lda].view(call.B, call.H, call.N, lda)
        ls = self.ls[:call.B * call.H * call.N * 2].view(call.B, call.H, call.N, 2)
        return a, ls

    def run(self, call, q, k, v, o, form):
        sd = self.sd
        scale = 1.0 / math.sqrt(call.d)
        if form == "flash":
            sd.flash(q, k, v, scale, out=o, ws=self.ws)
            return 1
        a, ls = self.views(call)
        if form == "three_pass":
            sd.qk_scores(q, k, scale, out_a=a)
            sd.row_stats(a, call.M, call.d, q.dtype, out_ls=ls, ws=self.ws)
            sd.softmax_av(a, ls, v, scale, out=o)
            return 3
        if form == "f16a":
            lda16 = (call.M + 7) // 8 * 8
            a16 = self.a.view(self.torch.float16)[:call.B * call.H * call.N * lda16]
            a16 = a16.view(call.B, call.H, call.N, lda16)
            sd.qk_stats_f16a(q, k, scale, out_a=a16, out_ls=ls, ws=self.ws)
            sd.softmax_av_f16a(a16, ls, v, scale, out=o)
            return 2
        sd.qk_stats(q, k, scale, out_a=a, out_ls=ls, ws=self.ws)
        sd.softmax_av(a, ls, v, scale, out=o)
        return 2


def run_gpu(args, rank, world, local_rank):
    import torch
    import diffusion_unet_attention_b200 as sd

    sd.load_library()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        from datetime import timedelta
        dist_mod.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
        dist = dist_mod

    stream = torch.cuda.Stream(device)
    sets = [StepSet(sd, torch, device, s) for s in range(2)]
    scratch = Scratch(sd, torch, device, CALLS)
    dom_calls = [i for i, c in enumerate(CALLS) if is_dominant(c)]
    rest_calls = [i for i, c in enumerate(CALLS) if not is_dominant(c)]

    def issue(stepset, idxs, form_of):
        n = 0
        for i in idxs:
            call, q, k, v, o = stepset.inputs[i]
            n += scratch.run(call, q, k, v, o, form_of(call))
        return n

    # ---- capture: per input set, the dominant segment and the rest ----------
    launches_per_step = 0
    graphs = []
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for s in sets:               # eager warm-up of every kernel variant before capture
            issue(s, range(len(CALLS)), policy_form)
        stream.synchronize()
        for s in sets:
            g_dom, g_rest = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_dom, stream=stream):
                n1 = issue(s, dom_calls, policy_form)
            with torch.cuda.graph(g_rest, stream=stream):
                n2 = issue(s, rest_calls, policy_form)
            graphs.append((g_dom, g_rest))
            launches_per_step = n1 + n2
    torch.cuda.synchronize()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    K, W = args.steps, args.warmup
    with torch.cuda.stream(stream):
        for i in range(W):
            g_dom, g_rest = graphs[i % 2]
            g_dom.replay()
            g_rest.replay()
    ev_dom = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(visible.split(",")[local_rank].strip() if visible else str(local_rank))
    barrier()
    clocks.start()
    time.sleep(0.3)
    wall0 = time.time()
    with torch.cuda.stream(stream):
        t0.record(stream)
        for i in range(K):
            g_dom, g_rest = graphs[i % 2]
            ev_dom[i][0].record(stream)
            g_dom.replay()
            ev_dom[i][1].record(stream)
            g_rest.replay()
        t1.record(stream)
    stream.synchronize()
    wall = time.time() - wall0
    barrier()
    clk = clocks.stop()
    elapsed_ms = t0.elapsed_time(t1)
    dom_ms = sum(a.elapsed_time(b) for a, b in ev_dom) / (K * len(dom_calls))
    elapsed_ms = max_over_ranks(elapsed_ms, dist, device)
    ms_per_step = elapsed_ms / K
    value = job_throughput(world, STEP_FLOPS, K, elapsed_ms)

    extra = {}
    e2e = None
    if rank == 0 and not args.no_side:
        extra = side_measurements(torch, sd, stream, sets, scratch, issue, K=min(K, 50))
        extra["per_call"] = per_call_table(torch, sd, stream, sets, scratch)
        extra["unet_ops"] = unet_ops_table(torch, sd, stream)
        extra["conv3x3_winograd"] = conv3x3_table(torch, sd, stream)
        extra["dtype_forms"] = dtype_forms_table(torch, sd, stream)
    if not args.no_side:
        # every rank feeds its own replica from host memory; the job's step is its slowest rank's
        barrier()
        e2e = end_to_end(torch, sd, stream, sets[0], scratch, steps=min(K, 20))
        e2e_ms = max_over_ranks(e2e["ms_per_step"], dist, device)
        e2e["ms_per_step"] = round(e2e_ms, 4)
        e2e["value"] = round(job_throughput(world, STEP_FLOPS, 1, e2e_ms), 3)

    peaks, peak_src = measured_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    dom_flops = synth.WORKLOADS["self64"].flops
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    traffic = profiled_traffic()
    line = {
        "metric": "attention us & TFLOP/s per UNet-step set (1xB200); % of tensor / HBM roofline",
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic N(0,1), seeded SplitMix64/Box-Muller, fp16",
        "config": job_config(world),
        "gpu_launches": launches_per_step * K,
        "roofline": {"bound": "tensor", "kernel": "flash_kernel<40,2,128> on 64x64 self-attention",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 dense burst (fp16 dense has the same nominal rate)",
                     "flops_per_launch": dom_flops, "avg_launch_us": round(dom_ms * 1e3, 3)},
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"],
                   "samples": clk["samples"], "power_w_median": clk.get("power_w_median")},
        "wall_s_timed": round(wall, 3),
    }
    if e2e is not None:
        line["e2e"] = e2e
    line.update(extra)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def side_measurements(torch, sd, stream, sets, scratch, issue, K):
    """Per-form step-set times and the two headline kernels on the 64x64
    self-attention, each timed with CUDA events (graph replays)."""
    out = {}

    def time_graph(build, reps, per_rep_div=1):
        gs = []
        with torch.cuda.stream(stream):
            for s in sets:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    build(s)
                gs.append(g)
            for i in range(3):
                gs[i % 2].replay()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(reps):
                gs[i % 2].replay()
            b.record(stream)
        stream.synchronize()
        del gs
        return a.elapsed_time(b) / reps / per_rep_div

    forms = {}
    for name, fn in (("flash_all", lambda c: "flash"), ("partial_all", lambda c: "partial"),
                     ("policy", policy_form)):
        ms = time_graph(lambda s, fn=fn: issue(s, range(len(CALLS)), fn), K)
        forms[name] = {"ms_per_step": round(ms, 5), "tflops": round(STEP_FLOPS / (ms * 1e-3) / 1e12, 2)}
    out["forms"] = forms

    # headline kernels on the 64x64 self-attention (5 distinct calls per replay)
    dom = [i for i, c in enumerate(CALLS) if is_dominant(c)]
    c2 = synth.WORKLOADS["self64"]
    peaks, _ = measured_peaks()
    f_ms = time_graph(lambda s: issue(s, dom, lambda c: "flash"), K, len(dom))
    p_ms = time_graph(lambda s: issue(s, dom, lambda c: "partial"), max(K // 4, 5), len(dom))
    t3_ms = time_graph(lambda s: issue(s, dom, lambda c: "three_pass"), max(K // 4, 5), len(dom))
    h_ms = time_graph(lambda s: issue(s, dom, lambda c: "f16a"), max(K // 4, 5), len(dom))
    io = 4 * c2.B * c2.H * c2.N * c2.d * 2 + c2.B * c2.H * c2.N * 8
    pf_bytes = 2 * c2.a_bytes() + io
    t3_bytes = 3 * c2.a_bytes() + io + c2.B * c2.H * c2.N * 8
    h_bytes = c2.a_bytes() + io
    out["kernels_64x64_self"] = {
        "flash": {"us": round(f_ms * 1e3, 2), "tflops": round(c2.flops / (f_ms * 1e-3) / 1e12, 1),
                  "frac_measured_tensor_peak": round(c2.flops / (f_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                  "frac_2250_tflops": round(c2.flops / (f_ms * 1e-3) / 2.25e15, 4)},
        "partially_fused": {"us": round(p_ms * 1e3, 2), "gbs": round(pf_bytes / (p_ms * 1e-3) / 1e9, 1),
                            "algorithmic_bytes": pf_bytes,
                            "frac_measured_hbm": round(pf_bytes / (p_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)},
        "three_pass": {"us": round(t3_ms * 1e3, 2), "gbs": round(t3_bytes / (t3_ms * 1e-3) / 1e9, 1),
                       "algorithmic_bytes": t3_bytes,
                       "frac_measured_hbm": round(t3_bytes / (t3_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                       "what": "qk_scores + row_stats (A read back) + softmax_av"},
        "f16a": {"us": round(h_ms * 1e3, 2), "gbs": round(h_bytes / (h_ms * 1e-3) / 1e9, 1),
                 "algorithmic_bytes": h_bytes,
                 "frac_measured_hbm": round(h_bytes / (h_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                 "what": "qk_stats_f16a + softmax_av_f16a (A stored in fp16)"},
    }
    return out


def per_call_table(torch, sd, stream, sets, scratch, reps=20):
    """Every distinct call of the step set in both forms, and each partially
    fused kernel alone: a CUDA graph of `reps` back-to-back launches of the
    call (the two input sets alternating, as within a step) is replayed and
    timed with CUDA events; time per call = replay time / reps.  Rows carry the
    call's algorithmic FLOPs and bytes, its fraction of the measured tensor
    (flash) or HBM (partially fused) peak, and its time over its floor: the
    larger of the FLOP floor, the byte floor and the time per launch of a
    minimal kernel timed the same way."""
    peaks, _ = measured_peaks()
    tflops_peak, hbm = float(peaks["bf16_tflops"]), float(peaks["hbm_gbs"])
    dev = sets[0].device
    tiny = torch.empty(4, dtype=torch.float32, device=dev)
    seen = {}
    for i, c in enumerate(CALLS):
        seen.setdefault((c.N, c.M, c.d), []).append(i)

    def per_launch_ms(issue_one):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for r in range(reps):
                    issue_one(r)
            for _ in range(2):
                g.replay()
            ts = []
            for _ in range(3):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g.replay()
                b.record(stream)
                stream.synchronize()
                ts.append(a.elapsed_time(b) / reps)
        del g
        return statistics.median(ts)

    launch_ms = per_launch_ms(lambda r: tiny.zero_())
    rows = []
    for (N, M, d), idxs in seen.items():
        i = idxs[0]
        call = CALLS[i]
        scale = 1.0 / math.sqrt(d)
        a, ls = scratch.views(call)
        inp = [sets[r % 2].inputs[i] for r in range(2)]

        def run(form):
            return lambda r: scratch.run(*inp[r % 2], form)

        f_ms = per_launch_ms(run("flash"))
        p_ms = per_launch_ms(run("partial"))
        qk_ms = per_launch_ms(lambda r: sd.qk_stats(inp[r % 2][1], inp[r % 2][2], scale, out_a=a, out_ls=ls,
                                                    ws=scratch.ws))
        av_ms = per_launch_ms(lambda r: sd.softmax_av(a, ls, inp[r % 2][3], scale, out=inp[r % 2][4]))
        io = 2 * call.B * call.H * (2 * call.N + 2 * call.M) * d          # Q, K, V read, O written
        pf_bytes = io + 2 * call.a_bytes() + 2 * 8 * call.B * call.H * call.N   # + A written, read; LS
        fl_floor = max(call.flops / (tflops_peak * 1e9), io / (hbm * 1e6), launch_ms)
        pf_floor = max(call.flops / (tflops_peak * 1e9), pf_bytes / (hbm * 1e6), 2 * launch_ms)
        rows.append({
            "call": call.name.split(" ", 1)[1], "N": N, "M": M, "d": d, "per_step": len(idxs),
            "policy": policy_form(call), "gflop": round(call.flops / 1e9, 3),
            "flash": {"us": round(f_ms * 1e3, 2), "tflops": round(call.flops / (f_ms * 1e-3) / 1e12, 1),
                      "frac_tensor": round(call.flops / (f_ms * 1e-3) / 1e12 / tflops_peak, 4),
                      "x_floor": round(f_ms / fl_floor, 2)},
            "partial": {"us": round(p_ms * 1e3, 2), "qk_stats_us": round(qk_ms * 1e3, 2),
                        "softmax_av_us": round(av_ms * 1e3, 2), "mb": round(pf_bytes / 1e6, 2),
                        "gbs": round(pf_bytes / (p_ms * 1e-3) / 1e9, 1),
                        "frac_hbm": round(pf_bytes / (p_ms * 1e-3) / 1e9 / hbm, 4),
                        "x_floor": round(p_ms / pf_floor, 2)},
        })
    return {"launch_floor_us": round(launch_ms * 1e3, 2),
            "note": f"graph replays of {reps} back-to-back launches of each call (two input sets alternating); "
                    "x_floor = time / max(FLOP floor, byte floor, minimal launch)", "rows": rows}


# The UNet's other specialised kernels at SD 1.4 512x512 shapes (B = 2):
# GroupNorm (32 groups) at the four resolutions, the gated GELU over
# 2 x h x w tokens with F = 4 x channels.
GN_SHAPES = [(2, 320, 64, 64), (2, 640, 32, 32), (2, 1280, 16, 16), (2, 1280, 8, 8)]
GEGLU_SHAPES = [(2 * 64 * 64, 1280), (2 * 32 * 32, 2560), (2 * 16 * 16, 5120), (2 * 8 * 8, 5120)]


def unet_ops_table(torch, sd, stream, reps=40):
    """GroupNorm and the gated GELU: each shape timed as a CUDA graph of `reps`
    launches cycling over enough input/output buffers that their total exceeds
    the L2 twice over (no launch finds its data in L2); bytes = input read once
    + output written once."""
    peaks, _ = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    dev = torch.device("cuda", torch.cuda.current_device())
    rows = []

    def timed(issue, nbuf):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for r in range(reps):
                    issue(r % nbuf)
            g.replay()
            ts = []
            for _ in range(3):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g.replay()
                b.record(stream)
                stream.synchronize()
                ts.append(a.elapsed_time(b) / reps)
        del g
        return statistics.median(ts)

    for (B, C, H, W) in GN_SHAPES:
        nbytes = 2 * 2 * B * C * H * W
        nbuf = max(2, math.ceil(256e6 / nbytes))
        xs = [torch.randn(B, C, H, W, device=dev, dtype=torch.float16) for _ in range(nbuf)]
        ys = [torch.empty_like(x) for x in xs]
        gam, bet = torch.ones(C, device=dev), torch.zeros(C, device=dev)
        ms = timed(lambda i: sd.group_norm(xs[i], gam, bet, 32, 1e-6, out=ys[i]), nbuf)
        rows.append({"op": "group_norm", "shape": [B, C, H, W], "groups": 32, "us": round(ms * 1e3, 2),
                     "mb": round(nbytes / 1e6, 2), "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                     "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4)})
        del xs, ys
    for (T, F) in GEGLU_SHAPES:
        nbytes = 2 * T * 2 * F + 2 * T * F
        nbuf = max(2, math.ceil(256e6 / nbytes))
        xs = [torch.randn(T, 2 * F, device=dev, dtype=torch.float16) for _ in range(nbuf)]
        ys = [torch.empty(T, F, device=dev, dtype=torch.float16) for _ in range(nbuf)]
        ms = timed(lambda i: sd.geglu(xs[i], out=ys[i]), nbuf)
        rows.append({"op": "geglu", "shape": [T, 2 * F], "us": round(ms * 1e3, 2), "mb": round(nbytes / 1e6, 2),
                     "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                     "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4)})
        del xs, ys
    return {"note": f"graph of {reps} launches over buffers totalling > 256 MB; fp16", "rows": rows}


CONV_SHAPES = [(2, 320, 64, 64), (2, 640, 32, 32), (2, 1280, 16, 16), (2, 1280, 8, 8)]


def conv3x3_table(torch, sd, stream, reps=20):
    """The UNet's 3x3 convolutions (C = K, 512x512 batch 2) by Winograd
    F(4x4, 3x3) against torch's convolution (cuDNN, an implicit-GEMM library
    kernel, autotuned), each as a CUDA graph of `reps` calls cycling over
    inputs and outputs that total more than twice the L2.  The filter is
    transformed once, outside the timed region (inference reuses it).
    Effective TFLOP/s counts the direct convolution's 2 * 9 * C * K * N * H * W;
    the Winograd path's bytes are x read, U read, V written and read, M
    (fp32) written and read, y written."""
    peaks, _ = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    dev = torch.device("cuda", torch.cuda.current_device())
    torch.backends.cudnn.benchmark = True
    rows = []

    def timed(issue, nbuf):
        for r in range(3):
            issue(r % nbuf)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for r in range(reps):
                    issue(r % nbuf)
            g.replay()
            ts = []
            for _ in range(3):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g.replay()
                b.record(stream)
                stream.synchronize()
                ts.append(a.elapsed_time(b) / reps)
        del g
        return statistics.median(ts)

    for (N, C, H, W) in CONV_SHAPES:
        K = C
        xbytes = 2 * N * C * H * W
        nbuf = max(2, math.ceil(256e6 / (2 * xbytes)))
        gen = torch.Generator(device=dev).manual_seed(C)
        xs = [torch.randn(N, C, H, W, device=dev, generator=gen).half() for _ in range(nbuf)]
        ys = [torch.empty(N, K, H, W, device=dev, dtype=torch.float16) for _ in range(nbuf)]
        w = (torch.randn(K, C, 3, 3, device=dev, generator=gen) / math.sqrt(9 * C)).half()
        bias = torch.randn(K, device=dev, generator=gen)
        bias16 = bias.half()
        U = sd.wino_filter(w)
        ws = torch.empty(sd.wino_workspace_bytes(N, C, K, H, W), dtype=torch.uint8, device=dev)
        with torch.cuda.stream(stream):
            ms_w = timed(lambda i: sd.conv3x3_winograd(xs[i], U, bias, out=ys[i], ws=ws), nbuf)
            ms_c = timed(lambda i: torch.nn.functional.conv2d(xs[i], w, bias16, padding=1), nbuf)
        T = N * ((H + 3) // 4) * ((W + 3) // 4)
        ldm = (T + 3) // 4 * 4
        path_bytes = xbytes + 36 * K * C * 2 + 2 * 36 * T * C * 2 + 2 * 36 * K * ldm * 4 + 2 * N * K * H * W
        flops = 2 * 9 * C * K * N * H * W
        rows.append({"shape": [N, C, H, W], "K": K, "winograd_us": round(ms_w * 1e3, 2), "cudnn_us": round(ms_c * 1e3, 2),
                     "speedup_vs_cudnn": round(ms_c / ms_w, 2), "direct_gflop": round(flops / 1e9, 2),
                     "eff_tflops": round(flops / (ms_w * 1e-3) / 1e12, 1),
                     "cudnn_tflops": round(flops / (ms_c * 1e-3) / 1e12, 1),
                     "winograd_path_mb": round(path_bytes / 1e6, 1),
                     "winograd_gbs": round(path_bytes / (ms_w * 1e-3) / 1e9, 1),
                     "frac_hbm": round(path_bytes / (ms_w * 1e-3) / 1e9 / hbm, 4)})
        del xs, ys, U, ws
    return {"note": f"graph of {reps} calls over buffers totalling > 256 MB; fp16, fp32 accumulation; filter "
                    "transformed once outside the timed region", "rows": rows}


def dtype_forms_table(torch, sd, stream, reps=20):
    """The forms for other input types: bf16 inputs with fp32 O (P carried in
    two 16-bit parts, two P V products), plain bf16 flash beside it, and fp32
    inputs through tf32 products, on the 64x64 self-attention and the tiny
    fp32 configuration.  Each is a graph of `reps` launches cycling over input
    sets that total more than 256 MB.  FLOPs are the algorithmic 4 B H N M d;
    the tf32 peak is the measured bf16 dense peak times the nominal
    tf32 / bf16 ratio (1.1 / 2.25 PFLOP/s)."""
    peaks, _ = measured_peaks()
    bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    dev = torch.device("cuda", torch.cuda.current_device())
    rows = []

    def timed(issue, nbuf):
        for r in range(3):
            issue(r % nbuf)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            with torch.cuda.graph(g, stream=stream):
                for r in range(reps):
                    issue(r % nbuf)
            g.replay()
            ts = []
            for _ in range(3):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g.replay()
                b.record(stream)
                stream.synchronize()
                ts.append(a.elapsed_time(b) / reps)
        del g
        return statistics.median(ts)

    cases = [("flash_f32o", "self64", torch.bfloat16), ("flash", "self64", torch.bfloat16),
             ("flash_tf32", "self64", torch.float32), ("flash_tf32", "tiny", torch.float32)]
    for form, wl, dtype in cases:
        c = synth.WORKLOADS[wl]
        per_set = c.B * c.H * (c.N + 2 * c.M) * c.d * (4 if dtype == torch.float32 else 2) + c.B * c.H * c.N * c.d * 4
        nbuf = max(2, math.ceil(256e6 / per_set))
        gen = torch.Generator(device=dev).manual_seed(c.d + c.N)
        sets = []
        for _ in range(nbuf):
            q = torch.randn(c.B, c.H, c.N, c.d, device=dev, generator=gen).to(dtype)
            k = torch.randn(c.B, c.H, c.M, c.d, device=dev, generator=gen).to(dtype)
            v = torch.randn(c.B, c.H, c.M, c.d, device=dev, generator=gen).to(dtype)
            o = torch.empty(c.B, c.H, c.N, c.d, device=dev,
                            dtype=dtype if form == "flash" else torch.float32)
            sets.append((q, k, v, o))
        scale = 1.0 / math.sqrt(c.d)
        fn = getattr(sd, form)
        with torch.cuda.stream(stream):
            ms = timed(lambda i: fn(sets[i][0], sets[i][1], sets[i][2], scale, out=sets[i][3]), nbuf)
        flops = 4 * c.B * c.H * c.N * c.M * c.d
        peak = bf16_peak * (1.1 / 2.25 if dtype == torch.float32 else 1.0)
        tflops = flops / (ms * 1e-3) / 1e12
        rows.append({"form": form, "workload": wl, "inputs": str(dtype).replace("torch.", ""),
                     "shape": [c.B, c.H, c.N, c.M, c.d], "us": round(ms * 1e3, 2), "tflops": round(tflops, 1),
                     "peak_tflops": round(peak, 1), "frac_peak": round(tflops / peak, 4)})
        del sets
    return {"note": f"graph of {reps} launches over inputs totalling > 256 MB; tf32 peak = measured bf16 x 1.1/2.25",
            "rows": rows}


def upload_groups(sizes, groups):
    """Consecutive runs of calls of about equal input bytes: [(first, end), ...]."""
    total = sum(sizes)
    out, start, acc = [], 0, 0
    for i, n in enumerate(sizes):
        acc += n
        if acc * groups >= total * (len(out) + 1) and len(out) < groups - 1:
            out.append((start, i + 1))
            start = i + 1
    if start < len(sizes):
        out.append((start, len(sizes)))
    return out


def end_to_end(torch, sd, stream, stepset, scratch, steps, groups=4):
    """The same metric through the public API with host buffers: every step
    copies the calls' inputs from pinned host memory, runs the set, and reads
    every O back.  The calls form `groups` consecutive runs of about equal
    input bytes; each run's Q, K, V travel host to device in one copy and its
    O's back in one copy (a few large copies keep the link busier than one per
    call while both directions run).  Copies in, calls and copies out run on
    three streams, so a run's calls overlap the next run's upload and the
    previous run's read-back; events keep each run's device buffers from being
    overwritten while in use."""
    inputs = stepset.inputs
    runs = upload_groups([q.numel() + k.numel() + v.numel() for _, q, k, v, _ in inputs], groups)
    host_in, dev_in, host_out, dev_out, views = [], [], [], [], []
    for r0, r1 in runs:
        flat = torch.cat([t.reshape(-1) for _, q, k, v, _ in inputs[r0:r1] for t in (q, k, v)]).cpu().pin_memory()
        dflat = torch.empty_like(flat, device=stream.device)
        oflat = torch.empty(sum(o.numel() for *_, o in inputs[r0:r1]), dtype=inputs[r0][4].dtype, device=stream.device)
        off = ooff = 0
        for call, q, k, v, o in inputs[r0:r1]:
            vq = dflat[off:off + q.numel()].view(q.shape)
            off += q.numel()
            vk = dflat[off:off + k.numel()].view(k.shape)
            off += k.numel()
            vv = dflat[off:off + v.numel()].view(v.shape)
            off += v.numel()
            vo = oflat[ooff:ooff + o.numel()].view(o.shape)
            ooff += o.numel()
            views.append((call, vq, vk, vv, vo))
        host_in.append(flat)
        dev_in.append(dflat)
        dev_out.append(oflat)
        host_out.append(torch.empty(oflat.shape, dtype=oflat.dtype).pin_memory())
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    n = len(runs)
    in_ready = [torch.cuda.Event() for _ in range(n)]    # run g's inputs are on the device
    done = [torch.cuda.Event() for _ in range(n)]        # run g's kernels have finished
    out_done = [torch.cuda.Event() for _ in range(n)]    # run g's O's are back on the host
    state = {"first": True}

    def one_step():
        first = state["first"]
        for g, (r0, r1) in enumerate(runs):
            with torch.cuda.stream(s_in):
                if not first:
                    s_in.wait_event(done[g])        # the previous step's kernels have read the run's inputs
                dev_in[g].copy_(host_in[g], non_blocking=True)
                in_ready[g].record(s_in)
            with torch.cuda.stream(stream):
                stream.wait_event(in_ready[g])
                if not first:
                    stream.wait_event(out_done[g])  # the previous step's read-back of the run's O's is complete
                for call, dq, dk, dv, do in views[r0:r1]:
                    scratch.run(call, dq, dk, dv, do, policy_form(call))
                done[g].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[g])
                host_out[g].copy_(dev_out[g], non_blocking=True)
                out_done[g].record(s_out)
        state["first"] = False

    one_step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_event(a)
    s_out.wait_event(a)
    for _ in range(steps):
        one_step()
    stream.wait_event(out_done[n - 1])
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    # every read-back equals what the device-resident inputs give under the same calls
    same = True
    with torch.cuda.stream(stream):
        for g, (r0, r1) in enumerate(runs):
            ooff = 0
            for call, q, k, v, o in inputs[r0:r1]:
                ref = torch.empty_like(o)
                scratch.run(call, q, k, v, ref, policy_form(call))
                got = host_out[g][ooff:ooff + o.numel()].view(o.shape)
                ooff += o.numel()
                same = same and torch.equal(got, ref.cpu())
    return {"value": round(STEP_FLOPS / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps, "outputs_match_device_run": same,
            "path": f"public Python API (ctypes -> C ABI), pinned host buffers, eager launches; the 32 calls in "
                    f"{n} consecutive runs, one upload (Q, K, V) and one read-back (O) per run, on three streams, "
                    f"overlapped across runs"}


# ----------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ----------------------------------------------------------------------------
class OracleSample:
    """The fp64 oracle on every `row_stride`-th query row of every call of the
    step set.  Inputs are drawn and widened to fp64 once; `run()` times only
    the oracle itself."""

    _inputs = None

    def __init__(self, row_stride: int):
        import oracle
        self.oracle = oracle
        self.lib = oracle.load()
        if OracleSample._inputs is None:
            cache = []
            for ci, call in enumerate(CALLS):
                q, k, v = synth.make_qkv(call, synth.STEP_SET_ID, call_id=ci)
                cache.append((call, q, np.ascontiguousarray(k, np.float64), np.ascontiguousarray(v, np.float64)))
            OracleSample._inputs = cache
        self.work = []
        self.flops = 0
        for call, q, k, v in OracleSample._inputs:
            qs = np.ascontiguousarray(q[:, :, ::row_stride], np.float64)
            self.work.append((qs, k, v, 1.0 / math.sqrt(call.d)))
            self.flops += 4 * call.B * call.H * qs.shape[2] * call.M * call.d
        self.stride = row_stride

    def run(self) -> float:
        t = time.perf_counter()
        for qs, k, v, scale in self.work:
            self.oracle.attention(qs, k, v, scale, lib=self.lib)
        return time.perf_counter() - t


def choose_stride(budget_s: float) -> int:
    """Row stride whose oracle sample takes about budget_s seconds."""
    probe = OracleSample(256)
    rate = probe.flops / max(probe.run(), 1e-6)
    return max(1, int(round(STEP_FLOPS * 1.0 / max(budget_s * rate, 1.0))))


def cpu_baseline(seconds: float):
    """The oracle on a row sample of the step set, repeated until about `seconds` of CPU work."""
    sample = OracleSample(choose_stride(seconds))
    s, n = sample.run(), 1
    while s < 0.8 * seconds and n < 16:
        s += sample.run()
        n += 1
    return {"value": round(n * sample.flops / s / 1e12, 6), "unit": "TFLOP/s", "cores": sample.oracle.max_threads(),
            "kind": "oracle",
            "sample": f"{n} x every {sample.stride}-th query row of all 32 calls of the step set "
                      f"({sample.flops / 1e9:.2f} GFLOP of the {STEP_FLOPS / 1e9:.1f} GFLOP step each time), "
                      f"fp64 C + OpenMP",
            "seconds": round(s, 2)}


def reference_stride(steps_total: int, budget_s: float = 150.0) -> int:
    """Row stride of each reference step: 1 (the whole step set) when
    `steps_total` whole steps fit in about `budget_s` seconds of oracle time,
    else the smallest stride whose sampled steps do."""
    probe = OracleSample(256)
    rate = probe.flops / max(probe.run(), 1e-6)
    full_s = STEP_FLOPS / rate
    return max(1, math.ceil(full_s * steps_total / budget_s))


def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle, as it stands, on the host cores,
    K timed steps after W untimed ones, each step the whole 32-call set when
    the run fits in a few minutes (else the same row sample of every call).
    `ms_per_step` is the measured time of one of those steps."""
    if rank != 0:
        return
    K, W = args.steps, args.warmup
    sample = OracleSample(reference_stride(K + W))
    for _ in range(W):
        sample.run()
    tot_s = 0.0
    for _ in range(K):
        tot_s += sample.run()
    value = sample.flops * K / tot_s / 1e12
    thr = sample.oracle.max_threads()
    what = ("the whole step set (all query rows of all 32 calls)" if sample.stride == 1 else
            f"every {sample.stride}-th query row of all 32 calls ({sample.flops / 1e9:.3f} of "
            f"{STEP_FLOPS / 1e9:.1f} GFLOP)")
    line = {"metric": "attention us & TFLOP/s per UNet-step set (1xB200); % of tensor / HBM roofline",
            "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": round(tot_s / K * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic N(0,1), seeded SplitMix64/Box-Muller, fp16 widened to fp64",
            "config": job_config(world), "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                             "sample": f"each step: {what}, fp64 C + OpenMP", "seconds": round(tot_s, 2)},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_case(args):
    """One form on one named workload, `reps` launches after one warm-up, each
    timed with CUDA events; used as the target of profiler captures."""
    import torch
    import diffusion_unet_attention_b200 as sd
    form, name = args.case.split(":")
    if form == "conv3x3":
        run_conv_case(args, torch, sd, name)
        return
    call = synth.WORKLOADS[name]
    device = torch.device("cuda", 0)
    q, k, v = synth.make_qkv(call, synth.STREAM[name])
    tq, tk, tv = (torch.from_numpy(x).to(device) for x in (q, k, v))
    o = torch.empty_like(tq)
    scratch = Scratch(sd, torch, device, [call])
    scale = 1.0 / math.sqrt(call.d)
    a, ls = scratch.views(call)
    # fp16-stored A: a view of the same scratch, rows of round_up(M, 8) halves
    lda16 = (call.M + 7) // 8 * 8
    a16 = scratch.a.view(torch.float16)[:call.B * call.H * call.N * lda16].view(call.B, call.H, call.N, lda16)

    def once():
        if form == "flash":
            sd.flash(tq, tk, tv, scale, out=o, ws=scratch.ws)
        elif form == "all":   # the three kernels of the step, one launch each
            sd.flash(tq, tk, tv, scale, out=o, ws=scratch.ws)
            sd.qk_stats(tq, tk, scale, out_a=a, out_ls=ls, ws=scratch.ws)
            sd.softmax_av(a, ls, tv, scale, out=o)
        elif form == "qk_stats":
            sd.qk_stats(tq, tk, scale, out_a=a, out_ls=ls, ws=scratch.ws)
        elif form == "softmax_av":
            sd.softmax_av(a, ls, tv, scale, out=o)
        elif form == "qk_stats_f16a":
            sd.qk_stats_f16a(tq, tk, scale, out_a=a16, out_ls=ls, ws=scratch.ws)
        elif form == "softmax_av_f16a":
            sd.softmax_av_f16a(a16, ls, tv, scale, out=o)
        elif form == "f16a":    # the fp16-A variant's two kernels
            sd.qk_stats_f16a(tq, tk, scale, out_a=a16, out_ls=ls, ws=scratch.ws)
            sd.softmax_av_f16a(a16, ls, tv, scale, out=o)
        elif form == "three_pass":    # A alone, the stand-alone reduction, softmax_av
            scratch.run(call, tq, tk, tv, o, "three_pass")
        else:
            scratch.run(call, tq, tk, tv, o, "partial")

    if form == "softmax_av":
        sd.qk_stats(tq, tk, scale, out_a=a, out_ls=ls, ws=scratch.ws)
    elif form == "softmax_av_f16a":
        sd.qk_stats_f16a(tq, tk, scale, out_a=a16, out_ls=ls, ws=scratch.ws)
    once()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        once()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    status = sd.device_error()
    print(json.dumps({"case": args.case, "shape": call.__dict__, "us": [round(t, 2) for t in times],
                      "device_error": status[0]}), flush=True)
    if status[0] != "SDATTN_OK":
        sys.exit(1)


def run_conv_case(args, torch, sd, name):
    """One of the UNet's 3x3 convolutions (`CxH`: batch 2, C = K channels,
    H = W) by Winograd: the filter transformed once, then `reps` timed calls
    after one warm-up, each with CUDA events."""
    C, H = (int(t) for t in name.split("x"))
    if (2, C, H, H) not in CONV_SHAPES:
        raise SystemExit(f"conv3x3 case {name}: not one of the UNet's shapes {CONV_SHAPES}")
    N, W, K = 2, H, C
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev).manual_seed(C)
    x = torch.randn(N, C, H, W, device=dev, generator=gen).half()
    w = (torch.randn(K, C, 3, 3, device=dev, generator=gen) / math.sqrt(9 * C)).half()
    bias = torch.randn(K, device=dev, generator=gen)
    U = sd.wino_filter(w)
    ws = torch.empty(sd.wino_workspace_bytes(N, C, K, H, W), dtype=torch.uint8, device=dev)
    y = torch.empty(N, K, H, W, device=dev, dtype=torch.float16)
    sd.conv3x3_winograd(x, U, bias, out=y, ws=ws)
    torch.cuda.synchronize()
    times = []
    for _ in range(args.reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        sd.conv3x3_winograd(x, U, bias, out=y, ws=ws)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    status = sd.device_error()
    print(json.dumps({"case": args.case, "shape": [N, C, H, W], "K": K, "us": [round(t, 2) for t in times],
                      "device_error": status[0]}), flush=True)
    if status[0] != "SDATTN_OK":
        sys.exit(1)


def main():
    args = parse_args()
    if args.case:
        run_case(args)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_gpu(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
