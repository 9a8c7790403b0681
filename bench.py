#!/usr/bin/env python
"""Throughput of the routed + shared-expert MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (one rank per GPU)

A step is one forward of the whole layer (router top-k, align/sort, stage 1,
stage 2 with the fused epilogue, and the side-stream shared expert) over one
batch of T tokens. The headline workload is the MXFP8 prefill layer (T=4096,
H=7168, E=256, top_k=8, I=2048, shared Is=2048, e4m3 with ue8m0 scales per 32
K elements, grouped sigmoid routing with a Zipf logit bias); the bf16 decode
layer (T=32, H=2048, E=128, top_k=8, I=768, Is=512, gated shared expert) is
measured in the same run and reported under "extra". Inputs and weights are
synthetic and seeded. The layer does not shard: under torchrun every rank runs
its own replica on its own GPU (weak scaling) and only the barrier and the
max-over-ranks timing cross ranks.

Timed region: exactly K steps replayed from CUDA graphs (both streams
captured), no timing events inside, inputs and weights resident in device
memory. Steps that read less than 3x the 126 MB L2 cycle through enough
independent weight copies that every step's weights come from HBM
(`config.l2`, `config.weight_copies`). Kernel durations for the roofline come
from the same graph with events around the two GEMMs, replayed once right
after the timed region. One JSON line is printed by rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from routed_shared_experts_b200 import configs, synth  # noqa: E402

METRIC = "MoE layer tokens/s"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "mxfp8_prefill"
EXTRA_WORKLOADS = "decode_bf16"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_WORKLOAD)
    ap.add_argument("--unroll", type=int, default=20, help="steps per captured graph")
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--extra", default=EXTRA_WORKLOADS,
                    help="comma-separated workloads measured after the headline and reported under 'extra' "
                         "('none' to skip)")
    ap.add_argument("--extra-min-steps", type=int, default=2000, help="at least this many steps per extra workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--nvtx", action="store_true",
                    help="mark the timed region with the NVTX range 'moe_steady_state' (for a launch list of it)")
    ap.add_argument("--router-gemm", action="store_true",
                    help="start each step from the router linear x . W_r (moe_router_gemm_topk) instead of logits")
    ap.add_argument("--fused-shared", action="store_true",
                    help="the shared expert as always-selected routed experts, one stream (FusedSharedMoELayer)")
    ap.add_argument("--quantize-x", action="store_true",
                    help="fp8/MXFP8 layers: start each step from bf16 x (moe_quantize_activations)")
    return ap.parse_args()


def workload_desc(cfg) -> str:
    return (f"{cfg.name}: T={cfg.T} H={cfg.H} E={cfg.E} top_k={cfg.top_k} I={cfg.I} Is={cfg.Is} "
            f"{cfg.dtype} {cfg.route}" + (" +gate" if cfg.shared_gate else ""))


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak(dtype: str):
    """Dense tensor-core peak (TFLOP/s) for the layer's GEMM operand type: the
    measured sustained bf16 cuBLAS figure (the bench times a long loop), times
    the nominal 2x of 8-bit over 16-bit operands for fp8 / MX layers."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        bf16, src = float(d.get("bf16_tflops_sustained") or d["bf16_tflops"]), "measured bf16 sustained"
    else:
        bf16, src = FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback bf16 sustained"
    if dtype == "bf16":
        return bf16, src
    return 2 * bf16, src + " x 2 (nominal 8-bit / 16-bit ratio)"


GEMM_SOURCES = ("gemm.cuh", "ptx.cuh", "moe_b200.cu")  # the GEMM kernels and the launcher that picks their instances


def _code_only(text: str) -> str:
    """C++ source without comments and blank lines: what the compiler sees."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())


def src_hash() -> str:
    """Hash of the GEMM kernels' code (comments left out, so that a counter
    taken on a kernel stays valid across edits of its comments only)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "routed_shared_experts_b200", "csrc")
    for f in GEMM_SOURCES:
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            h.update(f.encode() + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary, if it
    was taken on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rows = json.load(f)
    for r in rows:
        if r.get("kernel") == kernel and r.get("workload") == workload and r.get("src_sha") == src_hash():
            return r.get("dram_bytes_per_launch")
    return None


# ----------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons (100 ms period)."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        ident = None
        try:
            u = str(torch.cuda.get_device_properties(device).uuid)
            ident = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            ident = str(device)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={ident}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out = ""
        rows = []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 - 0.15 <= r[0] <= t1 + 0.15] or rows
        if not inside:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i in range(4) if r[3][i].lower().startswith("active")})
        sm = sorted(r[1] for r in inside)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside)}


# ----------------------------------------------------------------- helpers


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(v: float, world: int) -> float:
    """The largest of every rank's v (each rank's device time of the same
    region): the job is as slow as its slowest replica."""
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


L2_BYTES = 126e6


def l2_note(step_bytes: float, copies: int = 1) -> str:
    """How the step's bytes relate to the 126 MB L2 between timed steps."""
    if copies > 1:
        return (f"HBM: the step reads {step_bytes / 1e6:.1f} MB; steps cycle through {copies} weight copies "
                f"({copies * step_bytes / 1e6:.0f} MB, over 3x the 126 MB L2), so each step's weights come from HBM")
    return f"HBM: the step reads {step_bytes / 1e9:.2f} GB, over 3x the 126 MB L2, so weights come from HBM (no flush needed)"


def job_tokens_per_s(tokens_per_rank: int, world: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput of `world` replicas that each ran `steps` steps of
    `tokens_per_rank` tokens, timed as the slowest rank's `ms_max`."""
    return tokens_per_rank * world * steps / (ms_max / 1e3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def algorithmic_bytes(cfg, counts, router_gemm=False, quantize_x=False):
    """Bytes the layer and each GEMM must move at minimum (weights of the
    experts the routing activates, activations in and out once)."""
    active = int((counts > 0).sum())
    rows = int(counts.sum())
    w13 = synth.matrix_bytes(cfg.dtype, 2 * cfg.I * cfg.H)  # codes + scales
    w2 = synth.matrix_bytes(cfg.dtype, cfg.H * cfg.I)
    x = synth.activation_bytes(cfg.dtype, cfg.T, cfg.H)
    out = cfg.T * cfg.H * 2
    h = synth.activation_bytes(cfg.dtype, rows, cfg.I)
    s1 = active * w13 + x + h
    s2 = active * w2 + h + out + out + rows * 4  # h in, out, addend in, top-k weights
    shared = synth.shared_weight_bytes(cfg)
    layer = active * (w13 + w2) + shared + x + out + cfg.T * cfg.E * 4 + (cfg.H * 2 if cfg.shared_gate else 0)
    bf16_x_read = False
    if router_gemm:  # W_r and the bf16 x it multiplies (the logits are then written, not read)
        layer += cfg.H * cfg.E * 2
        bf16_x_read = cfg.dtype != "bf16"
    if quantize_x:  # bf16 x read, its codes written (then read as before)
        layer += cfg.T * cfg.H
        bf16_x_read = True
    if bf16_x_read:
        layer += cfg.T * cfg.H * 2
    # GEMM flops of the step (tensor-core work): every routed slot and every
    # token through the shared expert, gate_up (2I x H) and down (H x I)
    flops = 6 * rows * cfg.H * cfg.I + 6 * cfg.T * cfg.H * cfg.Is
    return {"active_experts": active, "stage1": s1, "stage2": s2, "layer": layer, "flops": flops}


# ----------------------------------------------------------------- our arm


def weight_copies(step_bytes: float) -> int:
    """Independent weight copies a run cycles through so that each step reads
    its weights from HBM: enough copies that consecutive uses of one copy are
    over 3x the L2 apart (the rotating-copies method of vllm-project/vllm PR
    65207, reviewer measurements "Commit 1": 12 layers cycling 6 weight
    copies)."""
    return max(1, math.ceil(3 * L2_BYTES / max(step_bytes, 1.0)))


WEIGHT_KEYS = ("w13", "w2", "w13s", "w2s", "w13_scale", "w2_scale", "w13s_scale", "w2s_scale", "w_gate")


def build_layers(cfg, inp, args, copies):
    """The layer and copies - 1 more whose weights are clones (activations
    and routing inputs shared, so every copy computes the same step)."""
    from routed_shared_experts_b200.layer import FusedSharedMoELayer, MoELayer

    def make(d):
        if args.fused_shared:
            return FusedSharedMoELayer(cfg, d)
        return MoELayer(cfg, d, router_gemm=args.router_gemm, quantize_x=args.quantize_x)
    layers = [make(inp)]
    for _ in range(copies - 1):
        d = dict(inp)
        for k in WEIGHT_KEYS:
            if d.get(k) is not None:
                d[k] = d[k].clone()
        layers.append(make(d))
    return layers


def measure(cfg, args, dev, world, steps, warmup, e2e_steps, clocks_local):
    """One workload: warm-up, then exactly `steps` steps replayed from CUDA
    graphs with no timing events inside (max over ranks), then the same graph
    shape with per-kernel timing events replayed once more for kernel
    durations, then the e2e serving loop with host buffers."""
    from routed_shared_experts_b200 import capi
    from routed_shared_experts_b200.pipeline import StepPipeline

    inp = synth.make_layer_inputs(cfg, device=dev)
    if args.router_gemm and cfg.dtype == "bf16":
        inp["x_r"] = inp["x"]  # the same bf16 activations feed the router linear and stage 1
    if args.fused_shared and (args.router_gemm or args.quantize_x):
        raise SystemExit("--fused-shared runs from logits and pre-quantised x")
    main = torch.cuda.Stream(device=dev)
    first = build_layers(cfg, inp, args, 1)[0]
    with torch.cuda.stream(main):
        first.forward(main)
    torch.cuda.synchronize()
    if capi.device_error(main) != 0:
        raise RuntimeError("device error after the first step")
    counts = first.expert_counts.cpu()[: cfg.E]  # routed experts (the fused layer appends the shared pieces)
    ab = algorithmic_bytes(cfg, counts, args.router_gemm, args.quantize_x)
    copies = weight_copies(ab["layer"])
    layers = [first] + (build_layers(cfg, inp, args, copies)[1:] if copies > 1 else [])

    # U steps per graph, a whole number of passes over the weight copies
    U = copies * max(1, math.ceil(min(args.unroll, steps) / copies))
    K = steps
    n_u, rem = divmod(K, U)
    probes = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(U)]

    def capture(n, probed=False):
        g = torch.cuda.CUDAGraph()
        main.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(main):
            with torch.cuda.graph(g, stream=main):
                for i in range(n):
                    layers[i % copies].forward(main, probes=probes[i] if probed else None)
        return g
    g_u = capture(U)
    g_r = capture(rem) if rem else None
    g_p = capture(U, probed=True)
    torch.cuda.synchronize()

    with torch.cuda.stream(main):
        for _ in range(max(1, math.ceil(warmup / U))):
            g_u.replay()
    torch.cuda.synchronize()

    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(clocks_local)
    time.sleep(0.3)  # let the sampler start
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    ev0.record(main)
    if args.nvtx:
        torch.cuda.nvtx.range_push("moe_steady_state")
    with torch.cuda.stream(main):
        for _ in range(n_u):
            g_u.replay()
        if g_r is not None:
            g_r.replay()
    if args.nvtx:
        torch.cuda.nvtx.range_pop()
    ev1.record(main)
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(world)
    clk = clocks.stop(t0, t1)
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    if capi.device_error(main) != 0:
        raise RuntimeError("device error in the timed region")

    # kernel durations: the probed graph (the same U steps with events around
    # the two GEMMs on the main stream), replayed right after the timed region
    with torch.cuda.stream(main):
        g_p.replay()
    torch.cuda.synchronize()

    def avg_us(a, b):
        return 1e3 * sum(p[a].elapsed_time(p[b]) for p in probes) / U
    s1_us, wait_us, s2_us = avg_us(0, 1), avg_us(1, 2), avg_us(2, 3)
    peak, peak_kind = peaks()
    tpeak, tpeak_src = tensor_peak(cfg.dtype)
    dom, dom_us = ("stage1", s1_us) if s1_us >= s2_us else ("stage2", s2_us)
    kname = "k_moe_gemm<stage1>" if dom == "stage1" else "k_moe_gemm<stage2>"
    achieved = ab[dom] / (dom_us * 1e-6) / 1e9
    traffic = recorded_traffic(kname, cfg.name)
    step_s = ms / 1e3 / K
    layer = layers[0]
    res = {
        "value": job_tokens_per_s(cfg.T, world, K, ms),
        "ms_per_step": ms / K,
        "steps": K,
        "dtype": cfg.dtype,
        "config": {"workload": workload_desc(cfg) + (" +router_gemm" if args.router_gemm else "")
                   + (" +quantize_x" if args.quantize_x else "") + (" +fused_shared" if args.fused_shared else ""),
                   "global_batch": cfg.T * world, "tokens_per_gpu": cfg.T, "parallelism": f"replicas{world}",
                   "l2": l2_note(ab["layer"], copies), "weight_copies": copies,
                   "graph": f"CUDA graphs of {U} steps, no timing events inside the timed region; kernel times from "
                            f"one probed replay of {U} steps right after it",
                   "block_m": layer.bm, "active_experts": ab["active_experts"]},
        "roofline": {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_kind, "traffic": traffic,
                     "bytes_per_launch": ab[dom], "launch_us": dom_us},
        "layer_roofline": {"bytes_per_step": ab["layer"], "t_roof_us": ab["layer"] / (peak * 1e9) * 1e6,
                           "t_step_us": step_s * 1e6, "frac": ab["layer"] / (peak * 1e9) / step_s,
                           "tensor": {"flops_per_step": ab["flops"], "peak_tflops": tpeak, "peak_source": tpeak_src,
                                      "t_roof_us": ab["flops"] / (tpeak * 1e12) * 1e6,
                                      "frac": ab["flops"] / (tpeak * 1e12) / step_s},
                           "binding": "hbm" if ab["layer"] / (peak * 1e9) >= ab["flops"] / (tpeak * 1e12)
                           else "tensor"},
        "kernels_us": {"stage1": s1_us, "addend_wait": wait_us, "stage2": s2_us,
                       "note": "one probed replay of the graph after the timed region"},
        "gpu_launches": K * layer.launches_per_step,
        "clocks": clk,
    }
    del g_u, g_r, g_p
    if e2e_steps <= 0:
        return res, inp

    # e2e through the serving loop (StepPipeline): every step copies its inputs
    # in from pinned host memory and its output back out, the copies of steps
    # i+1 and i-1 overlapping step i on a copy stream; eager C-ABI calls with
    # the same copies serialised for comparison
    names = ["x_r" if args.quantize_x else "x"]
    if not args.quantize_x and inp.get("x_scale") is not None:
        names.append("x_scale")
    if args.router_gemm:
        if cfg.dtype != "bf16" and not args.quantize_x:
            names.append("x_r")
    else:
        names.append("logits")
    hosts = [inp[n].cpu().pin_memory() for n in names]
    out_h = torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory()
    pipe = StepPipeline(layer, names, stream=main)
    outs = [out_h, torch.empty_like(out_h).pin_memory()]
    pipe.run([hosts] * 3, [outs[i % 2] for i in range(3)])
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e0.record(main)
    done = pipe.run([hosts] * e2e_steps, [outs[i % 2] for i in range(e2e_steps)])
    e1 = torch.cuda.Event(enable_timing=True)
    main.wait_event(done)
    e1.record(main)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    del pipe

    def eager_step():
        for n, hsrc in zip(names, hosts):
            inp[n].copy_(hsrc, non_blocking=True)
        layer.forward(main)
        out_h.copy_(layer.out, non_blocking=True)
    with torch.cuda.stream(main):
        for _ in range(3):
            eager_step()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(main)
    with torch.cuda.stream(main):
        for _ in range(e2e_steps):
            eager_step()
    e1.record(main)
    torch.cuda.synchronize()
    eager_ms = max_over_ranks(e0.elapsed_time(e1), world)
    res["e2e"] = {"value": job_tokens_per_s(cfg.T, world, e2e_steps, e2e_ms), "unit": UNIT,
                  "h2d_bytes_per_step": sum(hs.numel() * hs.element_size() for hs in hosts),
                  "d2h_bytes_per_step": out_h.numel() * out_h.element_size(), "steps": e2e_steps,
                  "api": "StepPipeline.run: per step H2D copies (pinned) -> graph of the step -> D2H copy (pinned), "
                         "the copies of steps i+1 and i-1 overlapping step i on a copy stream"
                         + ("" if copies == 1 else "; one weight copy (the device-timed value cycles "
                            f"{copies})"),
                  "eager": {"value": job_tokens_per_s(cfg.T, world, e2e_steps, eager_ms),
                            "api": "layer.forward() per step (eager C-ABI calls), the same copies serialised "
                                   "with it"}}
    return res, inp


def run_ours(args):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    cfg = configs.CONFIGS[args.config]
    res, inp = measure(cfg, args, dev, world, args.steps, args.warmup, args.e2e_steps, local)
    result = {
        "metric": METRIC,
        "value": res["value"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": res["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.dtype,
        "data": "synthetic",
    }
    for k in ("config", "roofline", "layer_roofline", "kernels_us", "e2e", "gpu_launches", "clocks"):
        if k in res:
            result[k] = res[k]
    extra = [w for w in (args.extra.split(",") if args.extra and args.extra != "none" else []) if w != args.config]
    if extra:
        result["extra"] = {}
        for name in extra:
            ecfg = configs.CONFIGS[name]
            steps = max(args.steps, args.extra_min_steps)
            r, _ = measure(ecfg, args, dev, world, steps, args.warmup, 0, local)
            result["extra"][name] = {k: r[k] for k in ("value", "ms_per_step", "steps", "dtype", "config", "roofline",
                                                        "layer_roofline", "kernels_us", "gpu_launches", "clocks")}
            result["gpu_launches"] += r["gpu_launches"]
        result["gpu_launches_note"] = "headline steps plus the extra workloads' steps"
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, synth.oracle_view(inp), min_s=10.0, max_s=30.0)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------- oracle


def cpu_baseline(cfg, inp, min_s: float, max_s: float):
    """The C++ oracle, as it stands, on the host threads: whole-token layer
    forwards (routing, shared expert with its gate, every routed expert, the
    one bf16 rounding) on a bounded subset of the workload's tokens, grown
    until min_s has passed (at most about max_s)."""
    import oracle
    c = cfg.as_dict()
    threads = oracle.num_threads()
    rng = np.random.default_rng(0)
    order = rng.permutation(cfg.T)
    done = 0
    n = threads
    t0 = time.time()
    while True:
        toks = order[done % cfg.T: done % cfg.T + n]
        oracle.moe_layer(c, inp, tokens=toks, threads=threads)
        done += len(toks)
        el = time.time() - t0
        per = el / done
        if el >= min_s or el + per * n > max_s:
            break
        n = max(threads, min(4 * threads, int((min_s - el) / per) // threads * threads))
    return {"value": done / el, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{done} of the workload's {cfg.T} tokens (seeded random subset), each a whole-layer forward "
                      f"through the plain C++ oracle (float64, OpenMP over tokens, {threads} threads), {el:.1f} s"}


def run_reference(args):
    """The oracle as the reference arm: each step is one batch of expert calls
    (one unit per host thread: a routed expert of one (token, slot) pair, or
    one token's shared expert; top_k + 1 units make one token), cycling
    through the workload's tokens."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from oracle import cpp
    cfg = configs.CONFIGS[args.config]
    inp = synth.oracle_view(synth.make_layer_inputs(cfg))
    threads = oracle.num_threads()
    lu = cpp.LayerUnits(cfg.as_dict(), inp, threads=threads)
    units = [(t, j) for t in range(cfg.T) for j in range(-1, cfg.top_k)]
    pos = 0

    def step():
        nonlocal pos
        batch = [units[(pos + i) % len(units)] for i in range(threads)]
        pos += threads
        lu.run(batch)

    for _ in range(args.warmup):
        step()
    t0 = time.time()
    for _ in range(args.steps):
        step()
    el = time.time() - t0
    tok = args.steps * threads / (cfg.top_k + 1)
    val = tok / el
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(cfg), "global_batch": cfg.T, "parallelism": "cpu"},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"each step = {threads} expert calls in parallel through the plain C++ oracle "
                                   f"(a routed expert of one (token, slot) pair or one token's shared expert; "
                                   f"{cfg.top_k + 1} calls = 1 token); {args.steps} steps"},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
