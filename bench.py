#!/usr/bin/env python
"""Benchmark of the MXFP4 MoE expert-MLP layer on B200 (one JSON line on stdout).

A step is one forward of the gpt-oss-20b-shaped MoE layer on the prefill
workload (T = 8192 tokens, H = I = 2880, 32 experts, top-4, MXFP4 expert
weights, W4A16): routing + gather, grouped gate/up GEMM with the SwiGLU
epilogue, grouped down GEMM with the routing weight, combine.  `value` is the
layer's algorithmic TFLOP/s, 2 * T * k * (2I*H + H*I) flops per step, with all
inputs resident in HBM.  The same JSON line also carries, measured in the same
run: quantize / dequantize GB/s on the bf16 [4096, 11520] tensor, the decode
layer (T = 64) as expert-weight GB/s, and the 120b-shaped layer (T = 4096,
128 experts) in W4A16 and W4A4 -- each against its roofline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 (torchrun, one process per GPU) every rank runs its own replica of
the layer on its own tokens (weak scaling, no collective on the data path);
time is the max over ranks.  `--impl reference` times the CPU oracle on the
host cores on a bounded sample of the same workload.
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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "MXFP4 MoE GEMM TFLOP/s & weight GB/s vs roofline; quantize GB/s (1 B200)"
L2_BYTES = 126 << 20          # B200 L2
KERNELS_PER_LAYER = {0: 6, 1: 8}   # W4A16: route x3, gate/up, down, combine; W4A4: + 2 quantize


# ------------------------------------------------------------------ environment

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def nvsmi_device_id(props) -> str:
    """The identifier nvidia-smi -i needs for a CUDA device, from its torch properties.

    A CUDA device index is logical (it counts only the devices CUDA_VISIBLE_DEVICES
    leaves visible), while nvidia-smi numbers every GPU of the machine, so the index
    can name another GPU.  The device UUID (else its PCI bus id) names the same GPU
    in both."""
    uuid = getattr(props, "uuid", None)
    if uuid:
        u = str(uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    return f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region (read-only
    queries of the GPU given by its nvidia-smi identifier, see nvsmi_device_id)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx_ = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        load = [v for v in sm if v > 0.5 * (max(mx_) if mx_ else 1)] or sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx_) if mx_ else None, "reasons": reasons,
                "samples": len(rows)}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """Max of v over all ranks (NCCL with a device tensor; gloo on the CPU)."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, steps: int, flops_per_step: float, total_ms_max: float) -> float:
    """Whole-job throughput in TFLOP/s: every rank runs `steps` steps of its own
    layer (replicas, weak scaling), timed by the slowest rank."""
    return world * steps * flops_per_step / total_ms_max / 1e9


# ------------------------------------------------------------------ workload set-up

def layer_flops(T, k, H, I):
    return 2.0 * T * k * (2 * I * H + H * I)


def gpu_layer(cfg, dev, T=None):
    """MoE layer inputs on the GPU; expert weights drawn per expert (seeded, fp32)
    and quantized to MXFP4 by the library's own quantize kernel."""
    import moe_expert_gemm_mxfp4_b200 as mx
    from moe_expert_gemm_mxfp4_b200 import inputs
    x, logits = inputs.moe_activations(cfg, T)
    E, H, I = cfg.E, cfg.H, cfg.I
    w13c = torch.empty((E, 2 * I, H // 2), dtype=torch.uint8, device=dev)
    w13s = torch.empty((E, 2 * I, H // 32), dtype=torch.uint8, device=dev)
    w2c = torch.empty((E, H, I // 2), dtype=torch.uint8, device=dev)
    w2s = torch.empty((E, H, I // 32), dtype=torch.uint8, device=dev)
    for e in range(E):
        w13, w2 = inputs.expert_weights(cfg, e)
        mx.mxfp4_quantize(w13.to(dev), codes=w13c[e], scales=w13s[e])
        mx.mxfp4_quantize(w2.to(dev), codes=w2c[e], scales=w2s[e])
    torch.cuda.synchronize()
    return dict(x=x, logits=logits, w=(w13c, w13s, w2c, w2s))


def make_events(n):
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record()
    torch.cuda.synchronize()
    return evs


def time_layer(L, cfg, mode, steps, warmup, dev, world=1, trace=True):
    """Device time of `steps` back-to-back layer calls (inputs resident).  No L2 flush:
    every call streams all expert weights (>= 423 MB, over 3x the L2), so a step
    finds at most the tail of the previous step's weights in L2.  Returns per-step ms,
    per-stage ms (gate/up, down, ...) and the outer wall."""
    import moe_expert_gemm_mxfp4_b200 as mx
    T = L["x"].shape[0]
    xd, ld = L["x"].to(dev), L["logits"].to(dev)
    out = torch.empty((T, cfg.H), dtype=torch.bfloat16, device=dev)
    ws = torch.empty((mx.moe_mxfp4_workspace_size(T, cfg.H, cfg.I, cfg.E, cfg.top_k, mode),),
                     dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        mx.moe_mxfp4_mlp(xd, ld, cfg.top_k, *L["w"], mode=mode, out=out, ws=ws)
    torch.cuda.synchronize()
    assert mx.mxfp4_get_device_status() == 0
    starts, ends = make_events(steps), make_events(steps)
    stage = [make_events(5) for _ in range(steps)] if trace else None
    outer0, outer1 = make_events(2)
    barrier(world)
    torch.cuda.synchronize()
    outer0.record()
    for i in range(steps):
        if trace:
            mx.mxfp4_set_trace_events(stage[i])
        starts[i].record()
        mx.moe_mxfp4_mlp(xd, ld, cfg.top_k, *L["w"], mode=mode, out=out, ws=ws)
        ends[i].record()
    outer1.record()
    torch.cuda.synchronize()
    barrier(world)
    mx.mxfp4_set_trace_events(None)
    assert mx.mxfp4_get_device_status() == 0
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    res = dict(step_ms=per_step, outer_ms=outer0.elapsed_time(outer1), out=out)
    if trace:
        names = ["route", "gate_up", "down", "combine"]
        res["stage_ms"] = {n: statistics.mean(st[j].elapsed_time(st[j + 1]) for st in stage)
                           for j, n in enumerate(names)}
    return res


def time_e2e(L, cfg, mode, steps, warmup, dev):
    """Same layer through the public API with host buffers: every step copies its x
    and router logits from pinned host memory to the device, runs the layer and copies
    the output back to pinned host memory, all inside the timing.  Device inputs and
    outputs are double-buffered so that one step's copies overlap another step's layer:
    H2D on one copy stream, D2H on another, the layer on the compute stream, ordered by
    events (a step's inputs land before its layer; a buffer is refilled only after the
    layer that read it, and an output buffer is rewritten only after its copy back).
    Returns (ms per step, H2D bytes per step, D2H bytes per step)."""
    import moe_expert_gemm_mxfp4_b200 as mx
    T = L["x"].shape[0]
    hx = L["x"].pin_memory()
    hl = L["logits"].pin_memory()
    hout = [torch.empty((T, cfg.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(hx, device=dev) for _ in range(2)]
    ld = [torch.empty_like(hl, device=dev) for _ in range(2)]
    out = [torch.empty((T, cfg.H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    ws = torch.empty((mx.moe_mxfp4_workspace_size(T, cfg.H, cfg.I, cfg.E, cfg.top_k, mode),),
                     dtype=torch.uint8, device=dev)
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    landed = [ev() for _ in range(2)]
    consumed = [ev() for _ in range(2)]
    fetched = [ev() for _ in range(2)]
    used = [False, False]

    def step(i):
        b = i & 1
        with torch.cuda.stream(up):
            if used[b]:
                up.wait_event(consumed[b])          # layer i-2 has read buffer b
            xd[b].copy_(hx, non_blocking=True)
            ld[b].copy_(hl, non_blocking=True)
            landed[b].record(up)
        comp.wait_event(landed[b])
        if used[b]:
            comp.wait_event(fetched[b])             # out[b] of step i-2 is back on the host
        mx.moe_mxfp4_mlp(xd[b], ld[b], cfg.top_k, *L["w"], mode=mode, out=out[b], ws=ws)
        consumed[b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(consumed[b])
            hout[b].copy_(out[b], non_blocking=True)
            fetched[b].record(down)
        used[b] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(up)
    for i in range(steps):
        step(warmup + i)
    down.wait_event(fetched[(warmup + steps - 1) & 1])
    z.record(down)
    torch.cuda.synchronize()
    return a.elapsed_time(z) / steps, hx.numel() * 2 + hl.numel() * 4, hout[0].numel() * 2


def time_kernel(fn, steps, warmup, dev):
    """Mean device time of fn(i), i = 0..steps-1; fn rotates over enough buffers that
    one call finds none of its data in L2.  A device-side spin is queued ahead of the
    timed calls: a kernel of a few tens of microseconds is shorter than the host's
    work to launch it, so without the spin each event pair would also bracket the
    device idling while the host prepares the launch.  With the device busy until
    the host has queued every call, each pair brackets its kernel alone."""
    for i in range(warmup):
        fn(i)
    torch.cuda.synchronize()
    s, e = make_events(steps), make_events(steps)
    torch.cuda._sleep(250_000 * steps)   # ~0.13 ms per timed call at 1.9 GHz
    for i in range(steps):
        s[i].record()
        fn(i)
        e[i].record()
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in zip(s, e))


# ------------------------------------------------------------------ breakdown lines

def bench_quant(dev, pk, steps=20, warmup=5):
    import moe_expert_gemm_mxfp4_b200 as mx
    from moe_expert_gemm_mxfp4_b200 import inputs
    x = inputs.quant_tensor().to(dev)
    R, C = x.shape
    codes = torch.empty((R, C // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((R, C // 32), dtype=torch.uint8, device=dev)
    out = torch.empty_like(x)
    nbytes = R * C * 2 + R * C // 2 + R * C // 32
    # copies of the 119 MB working set, cycled so that each call starts with its data
    # out of L2 (the L2 holds 126 MB; flushing it by writes instead would leave dirty
    # lines that the timed call then has to write back)
    nset = -(-2 * L2_BYTES // nbytes) + 1
    sets = [(x.clone(), torch.empty_like(codes), torch.empty_like(scales), torch.empty_like(out))
            for _ in range(nset)]
    tq = time_kernel(lambda i: mx.mxfp4_quantize(sets[i % nset][0], codes=sets[i % nset][1],
                                                 scales=sets[i % nset][2]), steps, warmup, dev)
    td = time_kernel(lambda i: mx.mxfp4_dequantize(sets[i % nset][1], sets[i % nset][2],
                                                   out=sets[i % nset][3]), steps, warmup, dev)
    gq, gd = nbytes / tq / 1e6, nbytes / td / 1e6
    return {"workload": f"bf16 [{R}, {C}] <-> MXFP4 (1% x50 outliers, 0.5% zero blocks)",
            "bytes_per_call": nbytes,
            "quantize": {"us": tq * 1e3, "gbs": gq, "frac_hbm": gq / pk["hbm"]},
            "dequantize": {"us": td * 1e3, "gbs": gd, "frac_hbm": gd / pk["hbm"]}}


def active_weight_bytes(cfg, logits):
    ids = torch.topk(logits, cfg.top_k, dim=1).indices.unique().numel()
    per_expert = (2 * cfg.I * cfg.H + cfg.H * cfg.I) * (0.5 + 1 / 32)
    return ids, ids * per_expert


# Nominal dense tensor peaks of a B200: fp4 9 PFLOP/s against bf16 2.25 PFLOP/s, the
# ratio used only when the live probe below has not run.
FP4_OVER_BF16 = 9.0 / 2.25


def measure_mma_rates(dev, iters=36000, reps=3):
    """Tensor-pipe rates of the library's two MMA kinds on this GPU, from its rate probe
    (one CTA per SM, back-to-back M = 128, N = 256 MMAs on random operands; ~10 ms per
    launch): best of `reps` launches each, in TFLOP/s, and their ratio mxf4 / f16."""
    import moe_expert_gemm_mxfp4_b200 as mx
    out = {}
    for kind, name in ((0, "f16"), (1, "mxf4")):
        mx.mxfp4_selftest_mma_rate(kind, 64)          # warm-up
        best = 0.0
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fl = mx.mxfp4_selftest_mma_rate(kind, iters)
            b.record()
            torch.cuda.synchronize()
            best = max(best, fl / a.elapsed_time(b) / 1e9)
        out[name + "_tflops"] = best
    assert mx.mxfp4_get_device_status() == 0
    out["mxf4_over_f16"] = out["mxf4_tflops"] / out["f16_tflops"]
    return out


def mxf4_peak(pk, rates=None):
    """Block-scaled fp4 (kind::mxf4) peak for the W4A4 roofline: the measured bf16 peak
    times the mxf4 / f16 rate ratio the probe measured on this GPU (else the nominal 4)."""
    if rates:
        return (pk["bf16"] * rates["mxf4_over_f16"],
                f"{pk['source']} bf16 x {rates['mxf4_over_f16']:.3f} (mxf4 / f16 tensor-pipe rate "
                f"ratio measured by the library's probe: {rates['mxf4_tflops']:.0f} / "
                f"{rates['f16_tflops']:.0f} TFLOP/s)")
    return pk["bf16"] * FP4_OVER_BF16, f"{pk['source']} bf16 x {FP4_OVER_BF16:g} (nominal dense fp4 / bf16)"


def w4a4_roofline(flops, weight_bytes, ms, pk, rates=None):
    """Roofline of a W4A4 layer: the slower of streaming its packed weights at the
    measured HBM bandwidth and its flops at the block-scaled fp4 peak; `frac` is that
    bound time over the measured time."""
    mxf4, src = mxf4_peak(pk, rates)
    hbm_us = weight_bytes / pk["hbm"] / 1e3
    mxf4_us = flops / mxf4 / 1e6
    bound_us = max(hbm_us, mxf4_us)
    return {"bound": "hbm" if hbm_us >= mxf4_us else "mxf4", "hbm_us": hbm_us, "mxf4_us": mxf4_us,
            "mxf4_peak_tflops": mxf4, "mxf4_peak_source": src,
            "bound_us": bound_us, "frac": bound_us / (ms * 1e3)}


def bench_moe_line(name, cfg, L, mode, dev, pk, steps=10, warmup=3, rates=None):
    r = time_layer(L, cfg, mode, steps, warmup, dev)
    ms = statistics.mean(r["step_ms"])
    fl = layer_flops(cfg.T, cfg.top_k, cfg.H, cfg.I)
    n_act, wbytes = active_weight_bytes(cfg, L["logits"])
    st = r["stage_ms"]
    line = {"workload": f"{name}: T={cfg.T} E={cfg.E} top-{cfg.top_k} H={cfg.H} I={cfg.I} "
                        f"{'W4A4' if mode else 'W4A16'}",
            "us_per_layer": ms * 1e3, "tflops": fl / ms / 1e9, "tokens_per_s": cfg.T / ms * 1e3,
            "active_experts": n_act, "weight_gbs": wbytes / ms / 1e6,
            "frac_hbm_weights": wbytes / ms / 1e6 / pk["hbm"],
            "frac_bf16": fl / ms / 1e9 / pk["bf16"],
            "stage_us": {k: v * 1e3 for k, v in st.items()}}
    gu_w = 2 * cfg.I * cfg.H * (0.5 + 1 / 32) * n_act
    dn_w = cfg.H * cfg.I * (0.5 + 1 / 32) * n_act
    line["gate_up"] = {"weight_gbs": gu_w / st["gate_up"] / 1e6,
                       "frac_hbm": gu_w / st["gate_up"] / 1e6 / pk["hbm"],
                       "tflops": fl * 2 / 3 / st["gate_up"] / 1e9,
                       "frac_bf16": fl * 2 / 3 / st["gate_up"] / 1e9 / pk["bf16"]}
    line["down"] = {"weight_gbs": dn_w / st["down"] / 1e6,
                    "frac_hbm": dn_w / st["down"] / 1e6 / pk["hbm"],
                    "tflops": fl / 3 / st["down"] / 1e9,
                    "frac_bf16": fl / 3 / st["down"] / 1e9 / pk["bf16"]}
    if mode == 1:   # W4A4
        line["roofline"] = w4a4_roofline(fl, wbytes, ms, pk, rates)
    return line


def bench_route_project(dev, steps=20, warmup=5):
    """Routing from the tokens (router projection fused with top-k, moe_mxfp4_route_project)
    against routing from precomputed logits (moe_mxfp4_route), per call, at the decode
    and prefill workloads' shapes.  Router weights bf16 [E, H] ~ N(0, 1/H)."""
    import moe_expert_gemm_mxfp4_b200 as mx
    from moe_expert_gemm_mxfp4_b200 import inputs
    out = {}
    for name in ("moe_decode", "moe_prefill"):
        cfg = inputs.MOE_CONFIGS[name]
        x, logits = inputs.moe_activations(cfg)
        x, logits, w = x.to(dev), logits.to(dev), inputs.router_weights(cfg).to(dev)
        ws = torch.empty((mx.moe_mxfp4_route_workspace_size(cfg.T, cfg.E, cfg.top_k),), dtype=torch.uint8,
                         device=dev)
        tp = time_kernel(lambda i: mx.moe_mxfp4_route_project(x, w, cfg.top_k, ws=ws), steps, warmup, dev)
        tr = time_kernel(lambda i: mx.moe_mxfp4_route(logits, cfg.top_k, ws=ws), steps, warmup, dev)
        proj_flops = 2.0 * cfg.T * cfg.E * cfg.H
        out[name] = {"T": cfg.T, "E": cfg.E, "H": cfg.H, "route_project_us": tp * 1e3,
                     "route_from_logits_us": tr * 1e3, "projection_tflops": proj_flops / tp / 1e9}
    assert mx.mxfp4_get_device_status() == 0
    return out


def bench_bf16_line(name, cfg, dev, pk, mxfp4_line=None, steps=10, warmup=3):
    """The same layer with bf16 expert weights (moe_bf16_mlp, the comparison the pages
    draw against MXFP4): per-layer time, weight GB/s and the MXFP4 layer's speed-up."""
    import moe_expert_gemm_mxfp4_b200 as mx
    from moe_expert_gemm_mxfp4_b200 import inputs
    E, H, I = cfg.E, cfg.H, cfg.I
    w13 = torch.empty((E, 2 * I, H), dtype=torch.bfloat16, device=dev)
    w2 = torch.empty((E, H, I), dtype=torch.bfloat16, device=dev)
    for e in range(E):
        a, b = inputs.expert_weights(cfg, e)
        w13[e].copy_(a.to(dev))
        w2[e].copy_(b.to(dev))
    x, logits = inputs.moe_activations(cfg)
    x, logits = x.to(dev), logits.to(dev)
    out = torch.empty((cfg.T, H), dtype=torch.bfloat16, device=dev)
    ws = torch.empty((mx.moe_bf16_workspace_size(cfg.T, H, I, E, cfg.top_k),), dtype=torch.uint8, device=dev)
    ms = time_kernel(lambda i: mx.moe_bf16_mlp(x, logits, cfg.top_k, w13, w2, out=out, ws=ws), steps, warmup, dev)
    assert mx.mxfp4_get_device_status() == 0
    n_act = torch.topk(logits, cfg.top_k, dim=1).indices.unique().numel()
    wbytes = n_act * (2 * I * H + H * I) * 2
    fl = layer_flops(cfg.T, cfg.top_k, H, I)
    line = {"workload": f"{name}: T={cfg.T} E={E} top-{cfg.top_k} H={H} I={I} bf16 weights",
            "us_per_layer": ms * 1e3, "tflops": fl / ms / 1e9, "weight_gbs": wbytes / ms / 1e6,
            "frac_hbm_weights": wbytes / ms / 1e6 / pk["hbm"], "frac_bf16": fl / ms / 1e9 / pk["bf16"],
            "weight_bytes": wbytes}
    if mxfp4_line:
        line["mxfp4_speedup"] = ms * 1e3 / mxfp4_line["us_per_layer"]
    del w13, w2
    torch.cuda.empty_cache()
    return line


def breakdown(dev, pk):
    import moe_expert_gemm_mxfp4_b200 as mx
    from moe_expert_gemm_mxfp4_b200 import inputs
    bd = {"quant": bench_quant(dev, pk)}
    bd["route_project"] = bench_route_project(dev)
    rates = measure_mma_rates(dev)
    bd["mma_probe"] = rates
    cfg = inputs.MOE_CONFIGS["moe_decode"]
    L = gpu_layer(cfg, dev)
    bd["moe_decode"] = bench_moe_line("moe_decode", cfg, L, mx.W4A16, dev, pk, steps=20)
    del L
    bd["moe_decode_bf16_weights"] = bench_bf16_line("moe_decode", cfg, dev, pk, bd["moe_decode"])
    cfg = inputs.MOE_CONFIGS["moe_120b"]
    L = gpu_layer(cfg, dev)
    bd["moe_120b_w4a16"] = bench_moe_line("moe_120b", cfg, L, mx.W4A16, dev, pk)
    bd["moe_120b_w4a4"] = bench_moe_line("moe_120b", cfg, L, mx.W4A4, dev, pk, rates=rates)
    del L
    torch.cuda.empty_cache()
    return bd


# ------------------------------------------------------------------ CPU oracle

def oracle_weights(cfg):
    import oracle
    from moe_expert_gemm_mxfp4_b200 import inputs
    E, H, I = cfg.E, cfg.H, cfg.I
    w13c = np.empty((E, 2 * I, H // 2), np.uint8)
    w13s = np.empty((E, 2 * I, H // 32), np.uint8)
    w2c = np.empty((E, H, I // 2), np.uint8)
    w2s = np.empty((E, H, I // 32), np.uint8)
    for e in range(E):
        w13, w2 = inputs.expert_weights(cfg, e)
        w13c[e], w13s[e] = oracle.quantize(w13.numpy(), oracle.FLOOR)
        w2c[e], w2s[e] = oracle.quantize(w2.numpy(), oracle.FLOOR)
    return w13c, w13s, w2c, w2s


def oracle_run(cfg, W, tokens):
    import oracle
    from moe_expert_gemm_mxfp4_b200 import inputs
    x, logits = inputs.moe_activations(cfg)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    t0 = time.perf_counter()
    oracle.moe_mlp(xb, logits.numpy(), cfg.top_k, *W, tokens=tokens)
    return time.perf_counter() - t0


def cpu_threads():
    return os.cpu_count() or 1


def cpu_baseline(cfg, n_tokens=16, seed=0):
    """The oracle, as it stands, on a seeded sample of the workload's tokens."""
    W = oracle_weights(cfg)
    g = torch.Generator().manual_seed(seed)
    tok = torch.randperm(cfg.T, generator=g)[:n_tokens].numpy()
    dt = oracle_run(cfg, W, tok)
    fl = layer_flops(n_tokens, cfg.top_k, cfg.H, cfg.I)
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{n_tokens} seeded tokens of the {cfg.T}-token layer (all their top-{cfg.top_k} "
                      f"experts: fp64 dequantize + fp64 matmuls), {dt:.1f} s wall"}


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle, K timed steps of one token each."""
    from moe_expert_gemm_mxfp4_b200 import inputs
    if rank != 0:
        return
    cfg = inputs.MOE_CONFIGS["moe_prefill"]
    W = oracle_weights(cfg)
    g = torch.Generator().manual_seed(1234)
    tok = torch.randperm(cfg.T, generator=g).numpy()
    for i in range(args.warmup):
        oracle_run(cfg, W, tok[i:i + 1])
    times = [oracle_run(cfg, W, tok[args.warmup + i:args.warmup + i + 1]) for i in range(args.steps)]
    dt = sum(times)
    fl = layer_flops(args.steps, cfg.top_k, cfg.H, cfg.I)
    v = fl / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": "each step: 1 seeded token of the 8192-token prefill layer "
                                       "(its 4 experts dequantized in fp64, fp64 matmuls)"},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(cfg):
    return {"workload": f"moe_prefill: gpt-oss-20b-shaped MoE expert-MLP layer, T={cfg.T} tokens, "
                        f"{cfg.E} experts, top-{cfg.top_k}, +2.0 router bias on experts 0-3, "
                        "MXFP4 weights, W4A16",
            "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "top_k": cfg.top_k,
            "flops_per_step": layer_flops(cfg.T, cfg.top_k, cfg.H, cfg.I),
            "l2": "inputs larger than L2, no flush: every step streams all 423 MB of expert "
                  "weights (126 MB L2); the quantize line cycles 3 copies of its 119 MB",
            "parallelism": "replicas (one layer per GPU, no collective)"}


def kernel_source_hash():
    """sha256[:16] over the sources of the grouped-GEMM kernels (a traffic figure
    is only reported while these are unchanged since it was captured)."""
    h = hashlib.sha256()
    for name in ("common.cuh", "gemm_common.cuh", "gemm.cu", "gemm_mxf4.cu"):
        with open(os.path.join(ROOT, "moe_expert_gemm_mxfp4_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current source of the kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        recs = json.load(f)
    h = kernel_source_hash()
    r = recs.get(f"{kernel}|{workload}")
    if not r or r.get("source_sha256_16") != h:
        return None
    return r.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ profiling driver

def run_profile_case(args):
    """The calls of one breakdown workload, for an ncu capture of its kernels."""
    import moe_expert_gemm_mxfp4_b200 as mx
    from moe_expert_gemm_mxfp4_b200 import inputs
    mx._lib.load()
    dev = torch.device("cuda", 0)
    n = args.warmup + args.steps
    if args.profile == "quant":
        x = inputs.quant_tensor().to(dev)
        for _ in range(n):
            c, sc = mx.mxfp4_quantize(x)
            mx.mxfp4_dequantize(c, sc)
    elif args.profile in ("route_project_decode", "route_project_prefill"):
        cfg = inputs.MOE_CONFIGS["moe_decode" if args.profile.endswith("decode") else "moe_prefill"]
        x, _ = inputs.moe_activations(cfg)
        x, w = x.to(dev), inputs.router_weights(cfg).to(dev)
        for _ in range(n):
            mx.moe_mxfp4_route_project(x, w, cfg.top_k)
    else:
        cfg = inputs.MOE_CONFIGS[{"decode": "moe_decode", "prefill": "moe_prefill"}.get(args.profile, "moe_120b")]
        if args.tokens:
            import dataclasses
            cfg = dataclasses.replace(cfg, T=args.tokens)
        mode = mx.W4A4 if args.profile == "w4a4_120b" else mx.W4A16
        L = gpu_layer(cfg, dev)
        xd, ld = L["x"].to(dev), L["logits"].to(dev)
        out = torch.empty((xd.shape[0], cfg.H), dtype=torch.bfloat16, device=dev)
        ws = torch.empty((mx.moe_mxfp4_workspace_size(xd.shape[0], cfg.H, cfg.I, cfg.E, cfg.top_k, mode),),
                         dtype=torch.uint8, device=dev)
        for _ in range(n):
            mx.moe_mxfp4_mlp(xd, ld, cfg.top_k, *L["w"], mode=mode, out=out, ws=ws)
    torch.cuda.synchronize()
    status = mx.mxfp4_get_device_status()
    print(json.dumps({"profile": args.profile, "calls": n, "device_status": status}), flush=True)
    if status != 0:
        sys.exit(1)


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-breakdown", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T of the prefill workload (profiling runs on a smaller case)")
    ap.add_argument("--profile", choices=["decode", "prefill", "w4a4_120b", "quant", "route_project_decode",
                                          "route_project_prefill"], default=None,
                    help="run one breakdown workload --warmup + --steps times, untimed, and "
                         "print a status line (a driver for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.profile:
        run_profile_case(args)
        return
    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    import moe_expert_gemm_mxfp4_b200 as mx
    from moe_expert_gemm_mxfp4_b200 import inputs
    mx._lib.load()   # fails loudly if the library is missing

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    pk = peaks()
    cfg = inputs.MOE_CONFIGS["moe_prefill"]
    if args.tokens:
        import dataclasses
        cfg = dataclasses.replace(cfg, T=args.tokens)
    L = gpu_layer(cfg, dev)

    sampler = ClockSampler(nvsmi_device_id(torch.cuda.get_device_properties(dev)))
    sampler.start()
    r = time_layer(L, cfg, mx.W4A16, args.steps, args.warmup, dev, world=world)
    clocks = sampler.stop()

    fl = layer_flops(cfg.T, cfg.top_k, cfg.H, cfg.I)
    step_ms = statistics.mean(r["step_ms"])
    total_ms = max_over_ranks(sum(r["step_ms"]), world)
    value = job_value(world, args.steps, fl, total_ms)
    st = r["stage_ms"]
    gu_flops = 2.0 * cfg.T * cfg.top_k * 2 * cfg.I * cfg.H
    achieved = gu_flops / st["gate_up"] / 1e9
    roof = {"kernel": "grouped_w4a16_kernel, gate/up projection + SwiGLU (192-row token tiles at this size)",
            "bound": "tensor", "achieved": achieved, "peak": pk["bf16"], "unit": "TFLOP/s",
            "frac": achieved / pk["bf16"],
            "peak_source": f"{pk['source']} bf16 dense (burst; timed region < 1 s)",
            "flops_per_launch": gu_flops,
            "traffic": traffic_record("grouped_w4a16_kernel_swiglu", "moe_prefill")}

    if rank != 0:
        barrier(world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    e2e_ms, h2d, d2h = time_e2e(L, cfg, mx.W4A16, max(3, args.steps // 2), 3, dev)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded torch CPU generator; weights ~N(0,0.02) quantized to MXFP4)",
            "config": workload_config(cfg),
            "tokens_per_s": world * args.steps * cfg.T / total_ms * 1e3,
            "stage_us": {k: v * 1e3 for k, v in st.items()},
            "roofline": roof,
            "e2e": {"value": fl / e2e_ms / 1e9, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": KERNELS_PER_LAYER[0] * args.steps,
            "clocks": clocks}
    del L
    torch.cuda.empty_cache()
    if not args.no_breakdown and world == 1:
        line["breakdown"] = breakdown(dev, pk)
        line["breakdown"]["moe_prefill_bf16_weights"] = bench_bf16_line(
            "moe_prefill", cfg, dev, pk, {"us_per_layer": step_ms * 1e3})
    if not args.no_cpu and world == 1:
        line["cpu_baseline"] = cpu_baseline(cfg)
    print(json.dumps(line), flush=True)
    if world > 1:
        barrier(world)
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
