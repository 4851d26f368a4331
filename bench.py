"""Benchmark of the MXFP4 MoE expert layer on B200 (one JSON line on rank 0).

A step is one moe_mxfp4_forward over one batch of synthetic tokens: router + top-k,
permute, expert gate_up + SwiGLU, down, weighted combine. Default workload (the line's
`value`): the largest single-GPU configuration, the 120B-shaped prefill layer with
Zipf(1.1)-skewed routing and FP8 activations (E=128, top-4, H=I=2880, T=16384, static
per-tensor scales from a 256-token calibration batch). In the same run, under
`other_configs`, the 120B prefill at T=4096 (uniform routing) and the 20B decode batches
T=1/8/64 (E=32, bf16 activations), each with its own step time, stage times, rooflines
and clocks. Other workloads (--workload): prefill, decode1/decode8/decode64,
prefill_bf16 (the prefill layer with bf16 activations), codec (the standalone MXFP4 codec
over the 120B-shaped expert set: a step is one quantize of all gate_up + down weights
from fp32 and one dequantize each to bf16 and fp32; metric GB/s of algorithmic bytes).

The FP8 tensor roofline divides by this GPU's measured rate for the MMA the prefill
GEMMs issue (the library's kind::mxf8f6f4 rate probe, run at the start of the bench).

Metric: MoE-layer tokens/s (whole job = sum over ranks). Inputs are resident in HBM
when the timed region starts; L2 is flushed before every timed step, outside the step's
own events: a 512 MiB write evicts it, a 256 MiB read leaves it holding clean lines of
an unrelated buffer (so the step does not pay the write-back of the flush). `e2e` is the same metric through the C ABI with the
tokens in pinned host memory: every step's host->device copy of x, the forward and the
device->host copy of the output are inside the timed region; the copies are double-
buffered on their own streams, so step i+1's copy in and step i-1's copy out overlap
step i's forward (as a serving loop would run them).

Multi-GPU (torchrun): every rank runs its own replica of the workload (the layer has no
cross-GPU exchange on this path), times are the max over ranks, value = total tokens of
all ranks / that time.

--impl reference: the CPU oracle on a bounded sample of the same workload, timed on the
host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mxfp4_block_scaled_moe_b200 import inputs  # noqa: E402

METRIC = "MoE-layer tokens/s"
CODEC_METRIC = "MXFP4 codec GB/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    # name: (constructor, fp8 activations)
    "prefill": (lambda dev: inputs.prefill_layer(T=4096, E=128, device=dev), True),
    "zipf": (lambda dev: inputs.zipf_layer(T=16384, E=128, device=dev), True),
    "prefill_bf16": (lambda dev: inputs.prefill_layer(T=4096, E=128, device=dev), False),
    "decode1": (lambda dev: inputs.decode_layer(T=1, E=32, device=dev), False),
    "decode8": (lambda dev: inputs.decode_layer(T=8, E=32, device=dev), False),
    "decode64": (lambda dev: inputs.decode_layer(T=64, E=32, device=dev), False),
}
CODEC = "codec"
CROSSOVER = "crossover"
ATTN = "attn_fp8"
# The default line: the largest single-GPU configuration (120B-shaped prefill, T = 16384,
# Zipf-skewed routing), then the 120B prefill at T = 4096 and the 20B decode batches
# measured in the same run.
DEFAULT_WORKLOAD = "zipf"
DEFAULT_EXTRAS = ("prefill", "decode1", "decode8", "decode64")

PER_EXPERT_PACKED = lambda H, I: 2 * I * H // 2 + 2 * I * H // 32 + H * I // 2 + H * I // 32


def ncu_traffic(workload: str, kernel: str):
    """Per-launch DRAM bytes (read + write) of `kernel` from a committed ncu summary under
    profiles/ (a block of "- key: value" lines starting at "- workload:"), or None when
    there is none or the kernel's source changed since."""
    import glob
    import hashlib
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        records, cur = [], None
        for line in open(path):
            line = line.strip()
            if not line.startswith("- ") or ": " not in line:
                continue
            k, v = line[2:].split(": ", 1)
            if k.strip() == "workload":
                cur = {}
                records.append(cur)
            if cur is not None:
                cur[k.strip()] = v.strip()
        for fields in records:
            if fields.get("workload") != workload or fields.get("kernel") != kernel:
                continue
            try:
                src, _, prefix = fields["source"].partition(" sha256 prefix ")
                digest = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()
                if not digest.startswith(prefix):
                    return None
                return int(fields["traffic_bytes_per_launch"])
            except (KeyError, OSError, ValueError):
                return None
    return None


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- distributed -----

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's time: every rank passes its own, all get the maximum."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank_step: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the tokens every rank processed over the slowest rank's time."""
    return tokens_per_rank_step * world * steps / (max_ms / 1e3)


# ----------------------------------------------------------------------- setup ----

def tensor_peak(B, seconds=1.0):
    """The FP8 block-scaled MMA rate of this GPU, measured with the library's rate probe
    (kind::mxf8f6f4, E4M3 x E2M1, M = 128, K = 32, one CTA per SM, operands resident in
    shared memory, pseudo-random operand bytes like a GEMM's data): `burst` = one ~10 ms
    launch on a GPU that has idled for a moment, `sustained` = the last second of
    back-to-back launches (the power cap's clock), both for N = 256, plus the prefill GEMM's
    own pattern (N = 240 with one scale-factor copy per four MMAs) at the sustained clock.
    Zero operands (which switch fewer bits and run faster under the power cap) are timed
    too, for reference. TFLOP/s."""
    stream = torch.cuda.current_stream()
    B.mxmoe_tc_rate_probe(256, False, 100)            # load the kernel
    torch.cuda.synchronize()
    time.sleep(0.5)

    def timed(n, copy, iters, rnd=True):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        f = B.mxmoe_tc_rate_probe(n, copy, iters, random_operands=rnd)
        e1.record(stream)
        return f, e0, e1

    def rate(r):
        return r[0] / (r[1].elapsed_time(r[2]) / 1e3) / 1e12

    zero = timed(256, False, 20000, rnd=False)      # from idle, as the burst below
    torch.cuda.synchronize()
    time.sleep(0.5)
    f, e0, e1 = timed(256, False, 20000)
    torch.cuda.synchronize()
    burst = f / (e0.elapsed_time(e1) / 1e3) / 1e12
    t_end = time.perf_counter() + seconds
    runs = []
    while time.perf_counter() < t_end:
        runs.append(timed(256, False, 20000))
        torch.cuda.synchronize()
    last = runs[-5:]
    sustained = sum(r[0] for r in last) / (sum(r[1].elapsed_time(r[2]) for r in last) / 1e3) / 1e12
    pat = timed(240, True, 20000)
    torch.cuda.synchronize()
    B.mxmoe_check()
    return {"peak_tflops": round(max(burst, sustained), 1),
            "burst_tflops": round(burst, 1), "sustained_tflops": round(sustained, 1),
            "n240_with_scale_copy_tflops": round(rate(pat), 1),
            "zero_operands_burst_tflops": round(rate(zero), 1),
            "probe": "tcgen05.mma kind::mxf8f6f4 block_scale, E4M3 x E2M1, M=128 N=256 K=32, "
                     "one CTA per SM, operands in shared memory: pseudo-random bytes (E4M3 "
                     "without NaN), unit scales"}


def layer_weights(lay, device, cache):
    """MXFP4 expert weights of a synthetic layer, quantized by the library's own kernel
    (cached per (E, H, I, seed): the prefill and Zipf layers share their experts)."""
    from mxfp4_block_scaled_moe_b200 import binding as B
    key = (lay.E, lay.H, lay.I, lay.seed)
    if key not in cache:
        E, H, I = lay.E, lay.H, lay.I
        gu_b = torch.empty(E, 2 * I, H // 2, dtype=torch.uint8, device=device)
        gu_s = torch.empty(E, 2 * I, H // 32, dtype=torch.uint8, device=device)
        d_b = torch.empty(E, H, I // 2, dtype=torch.uint8, device=device)
        d_s = torch.empty(E, H, I // 32, dtype=torch.uint8, device=device)
        for e in range(E):   # weights: fp32 draws quantized by the library's own kernel
            B.mxfp4_quantize(lay.gate_up(e), gu_b[e], gu_s[e])
            B.mxfp4_quantize(lay.down(e), d_b[e], d_s[e])
        cache[key] = (gu_b, gu_s, d_b, d_s)
    return cache[key]


def build_layer(name, device, cache=None):
    from mxfp4_block_scaled_moe_b200 import binding as B
    make, fp8 = WORKLOADS[name]
    lay = make(device)
    gu_b, gu_s, d_b, d_s = layer_weights(lay, device, {} if cache is None else cache)
    d = dict(x=lay.x, router_w=lay.router_w, router_b=lay.router_b, gu_blocks=gu_b,
             gu_scales=gu_s, gu_bias=lay.gu_bias, d_blocks=d_b, d_scales=d_s, d_bias=lay.d_bias)
    act = None
    if fp8:
        xc = inputs.calibration_x(H=lay.H, device=device)
        act = B.moe_mxfp4_calibrate(xc, lay.router_w, lay.router_b, gu_b, gu_s, lay.gu_bias,
                                    d_b, d_s, lay.d_bias, lay.k).cpu().tolist()
    torch.cuda.synchronize()
    return lay, d, act


def forward(B, d, k, act, out, stream=None):
    return B.moe_mxfp4_forward(d["x"], d["router_w"], d["router_b"], d["gu_blocks"],
                               d["gu_scales"], d["gu_bias"], d["d_blocks"], d["d_scales"],
                               d["d_bias"], k, act_scale=act, out=out, stream=stream)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed loop runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [c.strip() for c in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def algorithmic_work(lay, idx):
    """Bytes and FLOPs the step must move/do: packed weights of the distinct routed experts
    (+ biases), router weights, x in, out; FLOPs of the routed pairs and the router."""
    E, k, T, H, I = lay.E, lay.k, lay.T, lay.H, lay.I
    distinct = len(np.unique(idx.reshape(-1)))
    w_bytes = distinct * (PER_EXPERT_PACKED(H, I) + (2 * I + H) * 4)
    bytes_ = w_bytes + E * H * 2 + 2 * T * H * 2
    flops = T * k * (2 * H * 2 * I + 2 * I * H) + 2 * T * H * E
    gu_bytes = distinct * (2 * I * H // 2 + 2 * I * H // 32)
    gu_flops = T * k * 2 * H * 2 * I
    return dict(bytes=bytes_, flops=flops, distinct=distinct, gu_bytes=gu_bytes, gu_flops=gu_flops)


NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "fp8_tflops": 4500.0, "bf16_tflops": 2250.0}


def step_roofline(bytes_, flops, ms_per_step, pk, fp8, fp8_peak=None):
    """The whole step against the slower of its two bounds: algorithmic bytes over the HBM
    bandwidth and algorithmic FLOPs over the tensor peak (FP8 with FP8 activations, else
    bf16), with the measured peaks and the nominal ones. The measured FP8 peak is the rate
    probe's (fp8_peak, TFLOP/s); without it, 2x the measured bf16 peak (the nominal
    fp8/bf16 ratio). The measured bf16 peak is the burst figure. frac = that bound's time /
    the measured step time."""
    if fp8:
        meas_t = fp8_peak if fp8_peak else pk["bf16_tflops"] * 2.0
    else:
        meas_t = pk["bf16_tflops"]
    nom_t = NOMINAL_PEAKS["fp8_tflops" if fp8 else "bf16_tflops"]
    out = {}
    for name, bw, tp in (("measured", pk["hbm_gbs"], meas_t), ("nominal", NOMINAL_PEAKS["hbm_gbs"], nom_t)):
        t_mem = bytes_ / (bw * 1e9) * 1e3
        t_fl = flops / (tp * 1e12) * 1e3
        t = max(t_mem, t_fl)
        out[name] = {"bound": "hbm" if t_mem >= t_fl else "tensor", "hbm_gbs": bw, "tensor_tflops": tp,
                     "t_bound_ms": round(t, 5), "frac": round(t / ms_per_step, 4)}
    return out


# ------------------------------------------------------------- CPU baseline -----

def oracle_tokens_per_s(lay, d, act, budget_s, host_weights=None):
    """Time the oracle on a bounded prefix of the workload's tokens on the host cores."""
    import oracle
    hw = host_weights or {n: d[n].cpu().numpy() for n in
                          ("gu_blocks", "gu_scales", "gu_bias", "d_blocks", "d_scales", "d_bias")}
    xb = inputs.bits(d["x"])
    rw = inputs.bits(d["router_w"])
    rb = None if d["router_b"] is None else inputs.bits(d["router_b"])
    w = (hw["gu_blocks"], hw["gu_scales"], hw["gu_bias"], hw["d_blocks"], hw["d_scales"], hw["d_bias"])
    t0 = time.perf_counter()
    oracle.moe_forward(xb[:1], rw, rb, *w, lay.k, act_scale=act)
    t1 = time.perf_counter() - t0   # one token runs on one thread; tokens spread over cores
    n = int(max(1, min(lay.T, budget_s * oracle.num_threads() / max(t1, 1e-6))))
    t0 = time.perf_counter()
    oracle.moe_forward(xb[:n], rw, rb, *w, lay.k, act_scale=act)
    dt = time.perf_counter() - t0
    return n / dt, n, dt, hw


def oracle_one_token(lay, d, act):
    """The oracle on one token of the workload: its layer loop gives each token one thread,
    so this is the one-thread figure (tokens/s) beside the all-core cpu_baseline."""
    import oracle
    hw = {n: d[n].cpu().numpy() for n in ("gu_blocks", "gu_scales", "gu_bias", "d_blocks", "d_scales", "d_bias")}
    xb = inputs.bits(d["x"])
    rw = inputs.bits(d["router_w"])
    rb = None if d["router_b"] is None else inputs.bits(d["router_b"])
    w = (hw["gu_blocks"], hw["gu_scales"], hw["gu_bias"], hw["d_blocks"], hw["d_scales"], hw["d_bias"])
    oracle.moe_forward(xb[:1], rw, rb, *w, lay.k, act_scale=act)   # page the weights in
    t0 = time.perf_counter()
    oracle.moe_forward(xb[:1], rw, rb, *w, lay.k, act_scale=act)
    dt = time.perf_counter() - t0
    return {"value": round(1.0 / dt, 4), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"token 0 of the {lay.name} workload, {dt * 1e3:.0f} ms"}


# ------------------------------------------------------------------------ main ----

class L2Flush:
    """Evicts L2 between timed steps: a 512 MiB write, then a 256 MiB read that leaves L2
    holding clean lines of an unrelated buffer (so a step does not pay the flush's
    write-back)."""

    def __init__(self):
        self.flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
        self.clean = torch.zeros(32 << 20, dtype=torch.int64, device="cuda")     # 256 MiB
        self.clean_sum = torch.empty((), dtype=torch.int64, device="cuda")

    def __call__(self, i):
        self.flush.fill_(i & 0xFF)
        torch.sum(self.clean, dim=0, out=self.clean_sum)


def kernel_roofline(name, lay, work, stages, act, pk, pk_kind, tpk):
    """The dominant kernel (the largest stage other than routing, casts and combine)
    against its bound: tensor FLOPs at prefill sizes, packed-weight HBM bytes at decode
    (the whole step's bytes when the step is the one-launch decode layer)."""
    small = ("router", "topk", "router+topk", "route", "permute", "act_quant", "act_quant+scatter", "act_split",
             "mid_split", "combine")
    dom = max((s for s in stages if s not in small), key=lambda s: stages[s][0], default=None)
    if dom is None:
        dom = max(stages, key=lambda s: stages[s][0])
    dom_ms = stages[dom][0] / max(stages[dom][1], 1)
    fp8 = act is not None
    extra = {}
    if lay.T >= 1024:
        bound, unit = "tensor", "TFLOP/s"
        flops = work["gu_flops"] if dom == "gate_up" else work["flops"] if dom == "layer" else \
            work["flops"] - work["gu_flops"]
        achieved = flops / (dom_ms / 1e3) / 1e12
        if fp8 and tpk:
            peak = tpk["peak_tflops"]
            peak_note = "measured kind::mxf8f6f4 rate probe on random operands (this run, this GPU): the larger of burst and sustained"
            extra = {"frac_of_nominal_fp8": round(achieved / NOMINAL_PEAKS["fp8_tflops"], 4)}
        elif fp8:
            peak = pk["bf16_tflops"] * 2.0
            peak_note = f"{pk_kind} bf16 burst x 2 (nominal fp8/bf16 ratio)"
        else:
            # bf16 activations: a bf16 contraction (run as two e4m3 parts, the bf16 MMA rate)
            peak = pk["bf16_tflops"]
            peak_note = f"{pk_kind} bf16 burst (cuBLAS)"
            extra = {"frac_of_nominal_bf16": round(achieved / NOMINAL_PEAKS["bf16_tflops"], 4)}
    else:
        bound, unit = "hbm", "GB/s"
        peak = pk["hbm_gbs"]
        # "layer": the one-launch decode layer moves the whole step's bytes
        b = work["gu_bytes"] if dom == "gate_up" else work["bytes"] if dom == "layer" else \
            work["bytes"] - work["gu_bytes"]
        achieved = b / (dom_ms / 1e3) / 1e9
        peak_note = f"{pk_kind} hbm copy"
        extra = {"frac_of_nominal_hbm": round(achieved / NOMINAL_PEAKS["hbm_gbs"], 4)}
    r = {"bound": bound, "kernel": dom, "achieved": round(achieved, 2), "peak": peak,
         "unit": unit, "frac": round(achieved / peak, 4), "traffic": ncu_traffic(name, dom),
         "peak_source": peak_note, "kernel_ms": round(dom_ms, 5)}
    r.update(extra)
    return r


def measure_layer(B, name, lay, d, act, args, world, flusher, pk, pk_kind, tpk, with_e2e):
    """Device-timed steps of one workload (K steps in one CUDA graph, L2 flushed before
    each), per-stage times, rooflines, clocks; with_e2e adds the end-to-end leg."""
    k, T, H = lay.k, lay.T, lay.H
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    idx, _ = B.moe_route_topk(d["x"], d["router_w"], d["router_b"], k)
    work = algorithmic_work(lay, idx.cpu().numpy())

    for _ in range(args.warmup):
        forward(B, d, k, act, out)
    B.mxmoe_check()
    launches_per_step = B.mxmoe_last_launch_count()

    # ---- device-resident timed region: the K steps are captured into one CUDA graph as
    # [L2 flush, event, forward, event] x K and replayed once
    ev = [(torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True)) for _ in range(args.steps)]
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        forward(B, d, k, act, out)            # one more warm-up on the capture stream
    torch.cuda.synchronize()
    B.mxmoe_profile_enable(args.stage_events_in_timed_graph)
    with torch.cuda.graph(graph, stream=side):
        for i in range(args.steps):
            flusher(i)
            ev[i][0].record()
            forward(B, d, k, act, out)
            ev[i][1].record()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_end = time.perf_counter() + 1.0       # keep the GPU loaded while sampling starts
        while time.perf_counter() < t_end:
            graph.replay()
            torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("mxmoe_timed")
        graph.replay()                          # the timed region
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        barrier(world)
    stages = B.mxmoe_profile_read() if args.stage_events_in_timed_graph else {}
    B.mxmoe_profile_enable(False)
    B.mxmoe_check()
    total_ms = sum(a.elapsed_time(b) for a, b in ev)
    total_ms = max_over_ranks(total_ms, world)
    ms_per_step = total_ms / args.steps
    value = job_tokens_per_s(T, world, args.steps, total_ms)
    del graph

    e2e = None
    if with_e2e:
        e2e = e2e_leg(B, d, k, act, out, args, world)
    if not stages:   # stage times from an instrumented replay of the same graph shape
        B.mxmoe_profile_enable(True)
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=side):
            for i in range(args.steps):
                flusher(i)
                forward(B, d, k, act, out)
        torch.cuda.synchronize()
        g2.replay()
        torch.cuda.synchronize()
        stages = B.mxmoe_profile_read()
        B.mxmoe_profile_enable(False)
        del g2
    fp8 = act is not None
    res = {
        "value": round(value, 1), "ms_per_step": round(ms_per_step, 5),
        "roofline": kernel_roofline(name, lay, work, stages, act, pk, pk_kind, tpk),
        "step_roofline": step_roofline(work["bytes"], work["flops"], ms_per_step, pk, fp8,
                                       tpk["peak_tflops"] if (fp8 and tpk) else None),
        "stages_ms_per_step": {s: round(v[0] / max(v[1], 1), 5) for s, v in stages.items()},
        "algorithmic": {"bytes_per_step": work["bytes"], "flops_per_step": work["flops"],
                        "distinct_experts": work["distinct"]},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "config": {"workload": f"{name}: {lay.name}", "E": lay.E, "k": k, "T": T,
                   "H": H, "I": lay.I, "activations": "fp8_e4m3 static" if fp8 else "bf16",
                   "l2": "flushed before every timed step (512 MiB write, then a 256 MiB read)",
                   "parallelism": f"replicas x{world}"},
    }
    if e2e is not None:
        res["e2e"] = e2e
    return res


def _cpulist(text):
    cpus = set()
    for part in text.strip().split(","):
        if part:
            lo, _, hi = part.partition("-")
            cpus.update(range(int(lo), int(hi or lo) + 1))
    return cpus


def gpu_numa_cpus(dev):
    """(node, CPUs) of the NUMA node the GPU's PCI device sits on, the CPUs limited to those
    this process may run on; (None, None) when the topology is not visible."""
    try:
        p = torch.cuda.get_device_properties(dev)
        bdf = f"{p.pci_domain_id:04x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        node = int(open(f"/sys/bus/pci/devices/{bdf}/numa_node").read())
        if node < 0:
            return None, None
        cpus = _cpulist(open(f"/sys/devices/system/node/node{node}/cpulist").read()) & os.sched_getaffinity(0)
        return (node, cpus) if cpus else (None, None)
    except (OSError, ValueError, AttributeError):
        return None, None


def e2e_leg(B, d, k, act, out, args, world):
    """End to end through the C ABI with host buffers, double-buffered: the copy of the
    next step's tokens in and of the previous step's output out run on their own streams
    beside the current step's forward; every step's two copies are inside the timed region."""
    T, H = d["x"].shape
    stream = torch.cuda.current_stream()
    # pinned host buffers on the GPU's own NUMA node (a buffer on the other socket crosses
    # the inter-socket link on every copy): pages are placed where the allocating thread runs
    node, cpus = gpu_numa_cpus(torch.cuda.current_device())
    allowed = os.sched_getaffinity(0)
    if cpus:
        os.sched_setaffinity(0, cpus)
    try:
        x_host = d["x"].cpu().pin_memory()
        out_host = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    finally:
        os.sched_setaffinity(0, allowed)
    x_dev = [torch.empty_like(d["x"]) for _ in range(2)]
    out_dev = [torch.empty_like(out) for _ in range(2)]
    d_e2e = [dict(d, x=x_dev[s]) for s in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_done, fw_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def e2e_steps(n):
        for i in range(n):
            s = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(fw_done[s])     # forward i-2 has read x_dev[s]
                x_dev[s].copy_(x_host, non_blocking=True)
                in_done[s].record(s_in)
            stream.wait_event(in_done[s])
            if i >= 2:
                stream.wait_event(out_done[s])      # the copy out of step i-2 has read out_dev[s]
            forward(B, d_e2e[s], k, act, out_dev[s], stream=stream)
            fw_done[s].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(fw_done[s])
                out_host[s].copy_(out_dev[s], non_blocking=True)
                out_done[s].record(s_out)
        for s in range(min(n, 2)):
            stream.wait_event(out_done[s])          # the last copies out are inside the region

    e2e_steps(2)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    e2e_steps(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    return {"value": round(job_tokens_per_s(T, world, args.steps, e2e_ms), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 2,
            "host_numa_node": node,
            "timing": "steps back to back, copies double-buffered on their own streams, L2 not "
                      "flushed between steps (the routed experts' weights of a small batch can "
                      "stay in L2); pinned host buffers allocated on the GPU's NUMA node when "
                      "the topology is visible"}


def run_ours(args, world, rank):
    from mxfp4_block_scaled_moe_b200 import binding as B
    pk, pk_kind = peaks()
    cache = {}
    tpk = tensor_peak(B) if not args.no_tc_probe else None
    flusher = L2Flush()
    lay, d, act = build_layer(args.workload, "cuda", cache)
    head = measure_layer(B, args.workload, lay, d, act, args, world, flusher, pk, pk_kind, tpk, True)
    fp8 = act is not None
    res = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 x e2m1 -> f32" if fp8 else "bf16 x e2m1 -> f32",
        "data": "synthetic (seeded; weights N(0,0.02) quantized to MXFP4 on the GPU)",
        "config": head["config"],
        "roofline": head["roofline"],
        "step_roofline": head["step_roofline"],
        "stages_ms_per_step": head["stages_ms_per_step"],
        "algorithmic": head["algorithmic"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "timing": "K steps captured in one CUDA graph (flush, forward) and replayed once; "
                  "stage times from a replay of the same graph with per-stage events",
        "clocks": head["clocks"],
    }
    if tpk:
        res["tensor_peak_probe"] = tpk
    extras = [w for w in args.extra.split(",") if w and w != args.workload] if args.extra else []
    if extras:
        res["other_configs"] = {}
        for name in extras:
            lay2, d2, act2 = build_layer(name, "cuda", cache)
            r = measure_layer(B, name, lay2, d2, act2, args, world, flusher, pk, pk_kind, tpk, False)
            r["metric"], r["unit"] = METRIC, "tokens/s"
            if name == "decode1" and rank == 0 and world == 1 and not args.no_cpu_baseline:
                try:   # an auxiliary figure: its failure must not cost the line
                    r["cpu_baseline_1thread"] = oracle_one_token(lay2, d2, act2)
                except Exception as e:  # noqa: BLE001
                    r["cpu_baseline_1thread"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
            res["other_configs"][name] = r
            del lay2, d2
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n, dt, _ = oracle_tokens_per_s(lay, d, act, args.cpu_budget)
        import oracle
        res["cpu_baseline"] = {"value": round(v, 4), "unit": "tokens/s",
                               "cores": oracle.num_threads(), "kind": "oracle",
                               "sample": f"first {n} of {lay.T} tokens of the same workload, {dt:.1f} s"}
    return res


# --------------------------------------------- FP8 attention projections (fp8_linear) -----

ATTN_T = 4096
ATTN_SHAPES = (("qkv", 2880, 5120), ("o", 4096, 2880))   # (name, K in, N out)


def attn_weights(device):
    """FP8 E4M3 weights of the 120B model's attention projections with static per-tensor
    scales (min-max observer: s_w = amax / 448), drawn N(0, 0.02) and cast by the library."""
    from mxfp4_block_scaled_moe_b200 import binding as B
    ws = {}
    for name, K, N in ATTN_SHAPES:
        w = inputs.normal((N, K), 0.02, 0, "attn_" + name, 0, device)
        s_w = float(w.abs().max()) / 448.0
        wq = B.moe_fp8_quantize(w.to(torch.bfloat16), s_w)
        b = inputs.normal((N,), 0.01, 0, "attn_b_" + name, 0, device)
        ws[name] = (wq, s_w, b)
    torch.cuda.synchronize()
    return ws


def run_attn_fp8(args, world, rank):
    """A step = the fused Q/K/V projection (2880 -> 5120) and the O projection (4096 ->
    2880) of T tokens through fp8_linear (FP8 E4M3 weights and inputs, static per-tensor
    scales; "gpt-oss-120b-mxfp4-fp8attn-v2", Model Details). Metric tokens/s; roofline
    of the larger GEMM against the measured FP8 MMA rate (kind::f8f6f4 runs at the same
    rate as the probe's kind::mxf8f6f4, 16384 FLOP per SM cycle)."""
    from mxfp4_block_scaled_moe_b200 import binding as B
    pk, pk_kind = peaks()
    tpk = tensor_peak(B) if not args.no_tc_probe else None
    T = args.attn_tokens
    ws = attn_weights("cuda")
    xs = {name: inputs.normal((T, K), 1.0, 1, "attn_x_" + name, 0, "cuda", torch.bfloat16)
          for name, K, N in ATTN_SHAPES}
    s_x = {name: float(xs[name].float().abs().max()) / 448.0 for name, _, _ in ATTN_SHAPES}
    outs = {name: torch.empty(T, N, dtype=torch.bfloat16, device="cuda") for name, K, N in ATTN_SHAPES}
    flusher = L2Flush()

    def step():
        for name, K, N in ATTN_SHAPES:
            wq, s_w, b = ws[name]
            B.fp8_linear(xs[name], wq, s_x[name], s_w, b, out=outs[name])

    for _ in range(args.warmup):
        step()
    B.mxmoe_check()
    launches = 2 * len(ATTN_SHAPES)
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_end = time.perf_counter() + 1.0
        while time.perf_counter() < t_end:
            step()
            torch.cuda.synchronize()
        barrier(world)
        ms = time_steps(step, args.steps, flusher)
        barrier(world)
    ms = max_over_ranks(ms, world)
    per = {}
    for name, K, N in ATTN_SHAPES:
        wq, s_w, b = ws[name]
        per[name] = time_steps(lambda: B.fp8_linear(xs[name], wq, s_x[name], s_w, b, out=outs[name]),
                               args.steps, flusher)
    flops = {name: 2.0 * T * K * N for name, K, N in ATTN_SHAPES}
    dom = max(per, key=per.get)
    achieved = flops[dom] / (per[dom] / 1e3) / 1e12
    peak = tpk["peak_tflops"] if tpk else pk["bf16_tflops"] * 2.0
    res = {
        "metric": "FP8 attention-projection tokens/s", "value": round(T * world / (ms / 1e3), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 x e4m3 -> f32",
        "data": "synthetic (seeded; weights N(0,0.02) cast to FP8 E4M3 with a per-tensor min-max scale)",
        "config": {"workload": f"attn_fp8: fused QKV 2880->5120 and O 4096->2880, T={T}",
                   "l2": "flushed before every timed step (512 MiB write, then a 256 MiB read)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "kernel": f"fp8_linear {dom}", "achieved": round(achieved, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": None,
                     "peak_source": "measured kind::mxf8f6f4 rate probe on random operands (this run, this GPU)" if tpk
                     else f"{pk_kind} bf16 burst x 2", "kernel_ms": round(per[dom], 5),
                     "frac_of_nominal_fp8": round(achieved / NOMINAL_PEAKS["fp8_tflops"], 4)},
        "stages_ms_per_step": {k: round(v, 5) for k, v in per.items()},
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }
    if tpk:
        res["tensor_peak_probe"] = tpk
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        host = {name: (inputs.bits(xs[name]), ws[name][0].cpu().numpy(), ws[name][2].cpu().numpy())
                for name, _, _ in ATTN_SHAPES}

        def oracle_step(n):
            t0 = time.perf_counter()
            for name, K, N in ATTN_SHAPES:
                xb, wq_h, b_h = host[name]
                oracle.fp8_linear(xb[:n], wq_h, np.float32(s_x[name]), np.float32(ws[name][1]), b_h)
            return time.perf_counter() - t0

        t1 = oracle_step(1)   # one token per thread-slot: scale the sample to ~cpu_budget seconds
        n = int(max(1, min(T, args.cpu_budget * oracle.num_threads() / max(t1, 1e-6))))
        dt = oracle_step(n)
        res["cpu_baseline"] = {"value": round(n / dt, 4), "unit": "tokens/s", "cores": oracle.num_threads(),
                               "kind": "oracle", "sample": f"first {n} of {T} tokens, both projections, {dt:.1f} s"}
    return res


# ------------------------------------------------------- routed / dense crossover -----

CROSSOVER_GRID = ((32, 4, (16, 64, 128, 256, 512, 1024)), (128, 4, (64, 256, 512, 1024, 2048, 4096)),
                  (8, 8, (128, 1024, 4096)), (4, 4, (128, 1024, 4096)))


def time_steps(fn, steps, flusher):
    """Mean device time of one call of fn over `steps` calls captured in one CUDA graph,
    L2 flushed before each (CUDA events around every call)."""
    ev = [(torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True)) for _ in range(steps)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for i in range(steps):
            flusher(i)
            ev[i][0].record()
            fn()
            ev[i][1].record()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    del g
    return ms


def run_crossover(args, world, rank):
    """The routed path (moe_mxfp4_forward) against the dense all-experts path
    (moe_mxfp4_forward_dense) on the same layer, FP8 activations, uniform routing
    (router N(0, 1/sqrt(H))), H = I = 2880, over a grid of (E, k, T): top-4 of 32 and of
    128 experts, and k = E (every expert selected, where both paths do the same expert
    work). Reports both step times; the dense path does E/k times the expert work but needs
    no permutation, gather or scatter."""
    from mxfp4_block_scaled_moe_b200 import binding as B
    flusher = L2Flush()
    cache = {}
    rows = []
    for E, k, Ts in CROSSOVER_GRID:
        for T in Ts:
            lay = dataclasses.replace(inputs.prefill_layer(T=T, E=E, device="cuda"), k=k)
            gu_b, gu_s, d_b, d_s = layer_weights(lay, "cuda", cache)
            d = dict(x=lay.x, router_w=lay.router_w, router_b=lay.router_b, gu_blocks=gu_b, gu_scales=gu_s,
                     gu_bias=lay.gu_bias, d_blocks=d_b, d_scales=d_s, d_bias=lay.d_bias)
            xc = inputs.calibration_x(H=lay.H, device="cuda")
            act = B.moe_mxfp4_calibrate(xc, lay.router_w, lay.router_b, gu_b, gu_s, lay.gu_bias,
                                        d_b, d_s, lay.d_bias, lay.k).cpu().tolist()
            out = torch.empty(T, lay.H, dtype=torch.bfloat16, device="cuda")
            out_d = torch.empty_like(out)
            routed = lambda: forward(B, d, lay.k, act, out)
            dense = lambda: B.moe_mxfp4_forward_dense(d["x"], d["router_w"], d["router_b"], d["gu_blocks"],
                                                      d["gu_scales"], d["gu_bias"], d["d_blocks"], d["d_scales"],
                                                      d["d_bias"], lay.k, act_scale=act, out=out_d)
            for _ in range(args.warmup):
                routed()
                dense()
            B.mxmoe_check()
            t_r = time_steps(routed, args.steps, flusher)
            t_d = time_steps(dense, args.steps, flusher)
            B.mxmoe_check()
            same = bool(torch.equal(out.view(torch.int16), out_d.view(torch.int16))) if T > 64 else None
            rows.append({"E": E, "k": lay.k, "T": T, "routed_ms": round(t_r, 5), "dense_ms": round(t_d, 5),
                         "dense_over_routed": round(t_d / t_r, 3), "outputs_bit_identical": same})
            del d, lay
    return {"metric": "routed vs dense all-experts MoE-layer step time", "unit": "ms", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": False,
            "dtype": "e4m3 x e2m1 -> f32", "data": "synthetic (seeded; uniform routing)",
            "config": {"workload": "crossover: H = I = 2880, FP8 activations",
                       "l2": "flushed before every timed step"},
            "table": rows}


# ---------------------------------------------------------------- codec sweep -----

CODEC_H = 2880   # H = I = 2880: gate_up (E, 2I, H) and down (E, H, I) share K = 2880


def codec_sweep(n_experts, device):
    """The codec sweep's fp32 weights as ONE (rows, 2880) tensor: the gate_up rows of all
    experts (n_experts * 2I), then the down rows (n_experts * H). Both have K = 2880, and
    the codec treats a tensor as a flat run of 32-value blocks, so one launch per leg
    covers the whole set. Values: N(0, 0.02) with a Bernoulli(0.01) mask of outliers x 8
    (the same draws as the codec tests)."""
    K = CODEC_H
    rows_gu, rows_d = n_experts * 2 * K, n_experts * K
    w = torch.empty(rows_gu + rows_d, K, dtype=torch.float32, device=device)
    w[:rows_gu] = inputs.codec_tensor(rows_gu, K, seed=0, tag="gate_up", device=device)
    w[rows_gu:] = inputs.codec_tensor(rows_d, K, seed=0, tag="down", device=device)
    return w


def codec_leg_bytes(rows, K):
    """Algorithmic bytes of each codec leg over (rows, K) values: quantize reads fp32 and
    writes blocks + scales; dequantize reads blocks + scales and writes bf16 or fp32."""
    n = rows * K
    packed = n // 2 + n // 32
    return {"quantize": 4 * n + packed, "dequantize_bf16": packed + 2 * n,
            "dequantize_f32": packed + 4 * n}


def oracle_codec_gbs(w_host, budget_s):
    """The oracle's quantize + both dequantizes over the given rows, repeated until about
    budget_s seconds have passed; returns (GB/s, rows, repetitions, seconds)."""
    import oracle
    rows, K = w_host.shape
    reps = 0
    t0 = time.perf_counter()
    while True:
        blk, sc = oracle.quantize(w_host)
        oracle.dequantize(blk, sc, out="bf16")
        oracle.dequantize(blk, sc, out="f32")
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            break
    return sum(codec_leg_bytes(rows, K).values()) * reps / dt / 1e9, rows, reps, dt


def run_codec(args, world, rank):
    from mxfp4_block_scaled_moe_b200 import binding as B
    pk, pk_kind = peaks()
    w = codec_sweep(args.codec_experts, "cuda")
    torch.cuda.empty_cache()              # the draws' temporaries
    R, K = w.shape
    blocks = torch.empty(R, K // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(R, K // 32, dtype=torch.uint8, device="cuda")
    out16 = torch.empty(R, K, dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty(R, K, dtype=torch.float32, device="cuda")
    legs = [("quantize", lambda: B.mxfp4_quantize(w, blocks, scales)),
            ("dequantize_bf16", lambda: B.mxfp4_dequantize(blocks, scales, torch.bfloat16, out=out16)),
            ("dequantize_f32", lambda: B.mxfp4_dequantize(blocks, scales, torch.float32, out=out32))]
    leg_bytes = codec_leg_bytes(R, K)
    step_bytes = sum(leg_bytes.values())
    launches = 0
    for _ in range(args.warmup):
        for _, f in legs:
            f()
            launches += B.mxmoe_last_launch_count()
    B.mxmoe_check()
    launches_per_step = launches // max(args.warmup, 1)

    # every step reads 12.7 GB of fp32 and writes 19 GB: far larger than L2, no flush needed
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(legs) + 1)] for _ in range(args.steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        t_end = time.perf_counter() + 1.0
        while time.perf_counter() < t_end:
            for _, f in legs:
                f()
            torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("mxmoe_timed")
        for i in range(args.steps):
            ev[i][0].record()
            for j, (_, f) in enumerate(legs):
                f()
                ev[i][j + 1].record()
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        barrier(world)
    B.mxmoe_check()
    leg_ms = {n: sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps))
              for j, (n, _) in enumerate(legs)}
    total_ms = max_over_ranks(sum(leg_ms.values()), world)
    value = step_bytes * world * args.steps / (total_ms / 1e3) / 1e9
    dom = max(leg_ms, key=leg_ms.get)
    dom_ms = leg_ms[dom] / args.steps
    achieved = leg_bytes[dom] / (dom_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 2), "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4),
                "traffic": ncu_traffic(f"codec{args.codec_experts}", dom),
                "peak_source": f"{pk_kind} hbm copy", "kernel_ms": round(dom_ms, 5)}

    # ---- end to end through the C ABI from pinned host memory: the first experts' rows
    # in chunks of one expert's rows (gate_up or down); per chunk the fp32 rows go in,
    # the three legs run, and the packed, bf16 and fp32 results come back
    chunk = 2 * K
    rows_e2e = min(R, args.codec_e2e_chunks * chunk)
    node, cpus = gpu_numa_cpus(torch.cuda.current_device())   # pinned buffers near the GPU
    allowed = os.sched_getaffinity(0)
    if cpus:
        os.sched_setaffinity(0, cpus)
    try:
        w_host = w[:rows_e2e].cpu().pin_memory()
        blk_h = torch.empty(rows_e2e, K // 2, dtype=torch.uint8).pin_memory()
        sc_h = torch.empty(rows_e2e, K // 32, dtype=torch.uint8).pin_memory()
        o16_h = torch.empty(rows_e2e, K, dtype=torch.bfloat16).pin_memory()
        o32_h = torch.empty(rows_e2e, K, dtype=torch.float32).pin_memory()
    finally:
        os.sched_setaffinity(0, allowed)
    w_dev = torch.empty(chunk, K, dtype=torch.float32, device="cuda")

    def e2e_step():
        for r0 in range(0, rows_e2e, chunk):
            r1 = min(rows_e2e, r0 + chunk)
            n = r1 - r0
            w_dev[:n].copy_(w_host[r0:r1], non_blocking=True)
            B.mxfp4_quantize(w_dev[:n], blocks[:n], scales[:n])
            B.mxfp4_dequantize(blocks[:n], scales[:n], torch.bfloat16, out=out16[:n])
            B.mxfp4_dequantize(blocks[:n], scales[:n], torch.float32, out=out32[:n])
            blk_h[r0:r1].copy_(blocks[:n], non_blocking=True)
            sc_h[r0:r1].copy_(scales[:n], non_blocking=True)
            o16_h[r0:r1].copy_(out16[:n], non_blocking=True)
            o32_h[r0:r1].copy_(out32[:n], non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_bytes = sum(codec_leg_bytes(rows_e2e, K).values())
    e2e_value = e2e_bytes * world * args.steps / (e2e_ms / 1e3) / 1e9

    res = {
        "metric": CODEC_METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 -> e2m1 + e8m0 -> bf16 / f32",
        "data": "synthetic (seeded; N(0,0.02) with 1% outliers x 8)",
        "config": {"workload": f"codec: 120B-shaped expert set, {args.codec_experts} experts, "
                               f"gate_up ({args.codec_experts}, 5760, 2880) + down ({args.codec_experts}, 2880, 2880)",
                   "rows": R, "K": K, "values": R * K,
                   "l2": "not flushed: every step streams 12.7 GB in and 19 GB out at 128 experts, "
                         "far above the 126 MB L2",
                   "parallelism": f"replicas x{world}"},
        "roofline": roofline,
        "stages_ms_per_step": {n: round(v / args.steps, 5) for n, v in leg_ms.items()},
        "algorithmic": {"bytes_per_step": step_bytes, "bytes_per_leg": leg_bytes},
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s",
                "h2d_bytes_per_step": rows_e2e * K * 4,
                "d2h_bytes_per_step": rows_e2e * (K // 2 + K // 32 + 2 * K + 4 * K),
                "timing": f"the sweep's first {rows_e2e} rows in chunks of {chunk} from pinned host "
                          "memory; per chunk the copy in, the three legs and the four copies out run "
                          "in order on one stream"},
        "gpu_launches": launches_per_step * args.steps,
        "timing": "CUDA events around each leg of every step, K steps back to back",
    }
    res["clocks"] = clk.summary()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        v, rows, reps, dt = oracle_codec_gbs(w[: min(R, 1 << 16)].cpu().numpy(), args.cpu_budget)
        res["cpu_baseline"] = {"value": round(v, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                               "kind": "oracle",
                               "sample": f"first {rows} of {R} rows of the same sweep, {reps} passes "
                                         f"(quantize + both dequantizes) in {dt:.1f} s"}
    return res


def run_reference_codec(args, world, rank):
    """The oracle's codec over bounded row samples of the sweep, on the host cores."""
    if rank != 0:
        return None
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    K = CODEC_H
    # rows drawn like the sweep's gate_up rows (same recipe and seed)
    rows_all = args.codec_experts * 3 * K
    w = inputs.codec_tensor(min(rows_all, 1 << 14), K, seed=0, tag="gate_up", device=dev).cpu().numpy()
    oracle_codec_gbs(w, 0.0)                     # one untimed pass
    for _ in range(args.warmup - 1):
        oracle_codec_gbs(w, 0.0)
    t0 = time.perf_counter()
    reps = 0
    for _ in range(args.steps):                  # a step: passes over the sample for ~ref_step_s
        reps += oracle_codec_gbs(w, args.ref_step_s)[2]
    dt = time.perf_counter() - t0
    rows = w.shape[0]
    value = sum(codec_leg_bytes(rows, K).values()) * reps / dt / 1e9
    return {
        "impl": "reference", "metric": CODEC_METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 -> e2m1 + e8m0 -> bf16 / f32 (CPU oracle)",
        "data": "synthetic (seeded)",
        "config": {"workload": f"codec: 120B-shaped expert set, {args.codec_experts} experts",
                   "rows": rows_all, "K": K},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{rows} rows drawn like the sweep's, {reps} passes in {args.steps} steps"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def run_reference(args, world, rank):
    """The oracle as it stands, on the host cores, over bounded samples of the workload."""
    if rank != 0:
        return None
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    make, fp8 = WORKLOADS[args.workload]
    lay = make(dev)
    # pack with the oracle's own quantizer only the experts the sampled tokens route to
    xb, rw = inputs.bits(lay.x), inputs.bits(lay.router_w)
    rb = None if lay.router_b is None else inputs.bits(lay.router_b)
    E, H, I = lay.E, lay.H, lay.I
    hw = dict(gu_blocks=np.zeros((E, 2 * I, H // 2), np.uint8),
              gu_scales=np.full((E, 2 * I, H // 32), 127, np.uint8),
              gu_bias=lay.gu_bias.cpu().numpy(), d_blocks=np.zeros((E, H, I // 2), np.uint8),
              d_scales=np.full((E, H, I // 32), 127, np.uint8), d_bias=lay.d_bias.cpu().numpy())
    packed = set()

    def ensure(x_bits):
        idx, _ = oracle.topk_softmax(oracle.router_logits(x_bits, rw, rb), lay.k)
        for e in np.unique(idx):
            if e not in packed:
                hw["gu_blocks"][e], hw["gu_scales"][e] = oracle.quantize(lay.gate_up(int(e)).cpu().numpy())
                hw["d_blocks"][e], hw["d_scales"][e] = oracle.quantize(lay.down(int(e)).cpu().numpy())
                packed.add(e)

    act = None
    if fp8:
        xc = inputs.bits(inputs.calibration_x(H=H, device=dev))
        ensure(xc)
        act = oracle.calibrate(xc, rw, rb, hw["gu_blocks"], hw["gu_scales"], hw["gu_bias"],
                               hw["d_blocks"], hw["d_scales"], hw["d_bias"], lay.k)
    w = (hw["gu_blocks"], hw["gu_scales"], hw["gu_bias"], hw["d_blocks"], hw["d_scales"], hw["d_bias"])
    ensure(xb[:1])
    t0 = time.perf_counter()
    oracle.moe_forward(xb[:1], rw, rb, *w, lay.k, act_scale=act)
    t1 = time.perf_counter() - t0
    n = int(max(1, min(lay.T, args.ref_step_s * oracle.num_threads() / max(t1, 1e-6))))
    steps_rows = [np.arange(i * n, (i + 1) * n) % lay.T for i in range(args.warmup + args.steps)]
    for r in steps_rows:
        ensure(xb[r])
    for r in steps_rows[:args.warmup]:
        oracle.moe_forward(xb[r], rw, rb, *w, lay.k, act_scale=act)
    t0 = time.perf_counter()
    for r in steps_rows[args.warmup:]:
        oracle.moe_forward(xb[r], rw, rb, *w, lay.k, act_scale=act)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    sample = f"{n} tokens per step of the {lay.name} workload ({lay.T} tokens)"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 accumulate (CPU oracle)",
        "data": "synthetic (seeded)",
        "config": {"workload": f"{args.workload}: {lay.name}", "E": E, "k": lay.k, "T": lay.T,
                   "H": H, "I": I, "activations": "fp8_e4m3 static" if fp8 else "bf16"},
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + [CODEC, CROSSOVER, ATTN], default=DEFAULT_WORKLOAD)
    ap.add_argument("--attn-tokens", type=int, default=ATTN_T, help="attn_fp8 workload: tokens per step")
    ap.add_argument("--extra", default=None,
                    help="comma-separated workloads measured in the same run and reported under "
                         "other_configs (default: the 120B prefill and the three decode batches "
                         "with one GPU, none with several; '' for none)")
    ap.add_argument("--no-tc-probe", action="store_true",
                    help="skip the tensor-pipe rate probe (the FP8 roofline then uses 2x the "
                         "measured bf16 peak)")
    ap.add_argument("--codec-experts", type=int, default=128,
                    help="codec workload: experts of the 120B-shaped set to sweep")
    ap.add_argument("--codec-e2e-chunks", type=int, default=8,
                    help="codec workload: chunks of one expert's rows in the end-to-end leg")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    ap.add_argument("--ref-step-s", type=float, default=4.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stage-events-in-timed-graph", action="store_true",
                    help="record the library's per-stage events inside the timed graph itself "
                         "(they cost a few microseconds per stage); by default stage times come "
                         "from a separate replay of an instrumented copy of the graph")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.extra is None:
        single = int(os.environ.get("WORLD_SIZE", "1")) == 1
        args.extra = ",".join(DEFAULT_EXTRAS) if single and args.workload in WORKLOADS else ""
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if args.workload in (CROSSOVER, ATTN):
            res = {"impl": "reference", "unavailable": "the crossover and attention workloads report the oracle "
                                                       "as the cpu_baseline of their own line"}
            res = res if int(os.environ.get("RANK", "0")) == 0 else None
        else:
            res = (run_reference_codec if args.workload == CODEC else run_reference)(args, world, rank)
    else:
        world, rank = dist_init()
        try:
            run = {CODEC: run_codec, CROSSOVER: run_crossover, ATTN: run_attn_fp8}.get(args.workload, run_ours)
            res = run(args, world, rank)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
