#!/usr/bin/env python
"""Throughput of the routed + shared-expert MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (one rank per GPU)

A step is one forward of the whole layer (router top-k, align/sort, stage 1,
stage 2 with the fused epilogue, and the side-stream shared expert with its
gate) over one batch of T tokens of the decode workload (T=32, H=2048, E=128,
top_k=8, I=768, shared Is=512, bf16; synthetic seeded inputs and weights).
The layer does not shard: under torchrun every rank runs its own replica on its
own GPU (weak scaling) and only the barrier and the max-over-ranks timing cross
ranks.

Timed region: K steps replayed from CUDA graphs (both streams captured), with
the weights already resident in device memory. No L2 flush is done: for the
default workload the activated experts' weights (~0.8 GB per step) exceed the
126 MB L2, so every step reads them from HBM; `config.l2` states how each
workload's step bytes compare with the L2. The dominant kernel's duration is
taken from timing events captured inside the graph on its own stream. One JSON
line is printed by rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from routed_shared_experts_b200 import configs, synth  # noqa: E402

METRIC = "MoE layer tokens/s"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "decode_bf16"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_WORKLOAD)
    ap.add_argument("--unroll", type=int, default=20, help="steps per captured graph")
    ap.add_argument("--e2e-steps", type=int, default=300)
    ap.add_argument("--no-cpu-baseline", action="store_true")
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


def src_hash() -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "routed_shared_experts_b200", "csrc")
    for f in GEMM_SOURCES:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
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


def l2_note(step_bytes: float) -> str:
    """How the step's bytes relate to the 126 MB L2 between timed steps (no
    flush is done; the weights are not cycled through copies)."""
    if step_bytes >= 3 * L2_BYTES:
        return f"no flush: the step reads {step_bytes / 1e9:.2f} GB, over 3x the 126 MB L2, so weights come from HBM"
    if step_bytes > L2_BYTES:
        return (f"no flush: the step reads {step_bytes / 1e6:.0f} MB, 1-3x the 126 MB L2; part of the weights "
                "may still be in L2 from the previous step")
    return (f"no flush: the step reads {step_bytes / 1e6:.1f} MB, under the 126 MB L2, so the weights stay "
            "L2-resident across steps (launch-bound case, HBM roofline not meaningful)")


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


def run_ours(args):
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from routed_shared_experts_b200 import capi
    from routed_shared_experts_b200.layer import FusedSharedMoELayer, MoELayer
    from routed_shared_experts_b200.pipeline import StepPipeline

    cfg = configs.CONFIGS[args.config]
    inp = synth.make_layer_inputs(cfg, device=dev)
    if args.router_gemm and cfg.dtype == "bf16":
        inp["x_r"] = inp["x"]  # the same bf16 activations feed the router linear and stage 1
    if args.fused_shared:
        if args.router_gemm or args.quantize_x:
            raise SystemExit("--fused-shared runs from logits and pre-quantised x")
        layer = FusedSharedMoELayer(cfg, inp)
    else:
        layer = MoELayer(cfg, inp, router_gemm=args.router_gemm, quantize_x=args.quantize_x)
    main = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(main):
        layer.forward(main)
    torch.cuda.synchronize()
    if capi.device_error(main) != 0:
        raise RuntimeError("device error after the first step")
    counts = layer.expert_counts.cpu()[: cfg.E]  # routed experts (the fused layer appends the shared pieces)
    ab = algorithmic_bytes(cfg, counts, args.router_gemm, args.quantize_x)

    # graphs: U unrolled plain steps, the same U steps with timing events
    # around the two GEMMs (events inside a graph add a few microseconds each,
    # so only the last U steps of the timed region carry them), and one plain
    # step for the remainder
    U = max(1, min(args.unroll, args.steps))
    probes = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(U)]
    g_u = torch.cuda.CUDAGraph()
    g_p = torch.cuda.CUDAGraph()
    g_1 = torch.cuda.CUDAGraph()
    main.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(main):
        with torch.cuda.graph(g_u, stream=main):
            for _ in range(U):
                layer.forward(main)
        with torch.cuda.graph(g_p, stream=main):
            for i in range(U):
                layer.forward(main, probes=probes[i])
        with torch.cuda.graph(g_1, stream=main):
            layer.forward(main)
    torch.cuda.synchronize()

    with torch.cuda.stream(main):
        for _ in range(args.warmup):
            g_1.replay()
    torch.cuda.synchronize()

    K = args.steps
    n_u, rem = divmod(K - U, U) if K >= U else (0, K)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    time.sleep(0.3)  # let the sampler start
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    ev0.record(main)
    with torch.cuda.stream(main):
        for _ in range(rem):
            g_1.replay()
        for _ in range(n_u):
            g_u.replay()
        if K >= U:
            g_p.replay()
    ev1.record(main)
    torch.cuda.synchronize()
    t1 = time.time()
    barrier(world)
    clk = clocks.stop(t0, t1)
    ms = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms, world)
    if capi.device_error(main) != 0:
        raise RuntimeError("device error in the timed region")

    # per-kernel durations of the last U launches inside the timed region
    def avg_us(a, b):
        return 1e3 * sum(p[a].elapsed_time(p[b]) for p in probes) / U if K >= U else float("nan")
    s1_us, wait_us, s2_us = avg_us(0, 1), avg_us(1, 2), avg_us(2, 3)
    peak, peak_kind = peaks()
    tpeak, tpeak_src = tensor_peak(cfg.dtype)
    dom, dom_us = ("stage1", s1_us) if s1_us >= s2_us else ("stage2", s2_us)
    kname = "k_moe_gemm<stage1>" if dom == "stage1" else "k_moe_gemm<stage2>"
    achieved = ab[dom] / (dom_us * 1e-6) / 1e9
    traffic = recorded_traffic(kname, cfg.name)
    step_s = ms / 1e3 / K

    # e2e with host buffers, every step: H2D of the step's inputs from pinned
    # memory, the step, D2H of its output (StepPipeline below; eager for comparison)
    # step inputs copied from pinned host memory: the activations the step
    # reads (bf16 x when the step quantises it, else x in the layer's format),
    # and the logits unless the step starts from the router linear, which
    # reads bf16 x (the same tensor for a bf16 layer or with --quantize-x)
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
    E2E = args.e2e_steps

    def e2e_run(step):
        """E2E steps of: H2D copies of the inputs, one layer step, D2H copy of
        the output, all on the main stream; device time between two events."""
        with torch.cuda.stream(main):
            for _ in range(3):
                for n, hsrc in zip(names, hosts):
                    inp[n].copy_(hsrc, non_blocking=True)
                step()
                out_h.copy_(layer.out, non_blocking=True)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(main)
        with torch.cuda.stream(main):
            for _ in range(E2E):
                for n, hsrc in zip(names, hosts):
                    inp[n].copy_(hsrc, non_blocking=True)
                step()
                out_h.copy_(layer.out, non_blocking=True)
        e1.record(main)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), world)

    # the serving path (StepPipeline): every step's inputs copied in and its
    # output copied out, the copies of neighbouring steps overlapping the step
    pipe = StepPipeline(layer, names, stream=main)
    outs = [out_h, torch.empty_like(out_h).pin_memory()]
    pipe.run([hosts] * 3, [outs[i % 2] for i in range(3)])
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e0.record(main)
    done = pipe.run([hosts] * E2E, [outs[i % 2] for i in range(E2E)])
    e1 = torch.cuda.Event(enable_timing=True)
    main.wait_event(done)
    e1.record(main)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    del pipe
    eager_ms = e2e_run(lambda: layer.forward(main))  # one step at a time, eager C-ABI calls, serial copies
    barrier(world)

    result = {
        "metric": METRIC,
        "value": job_tokens_per_s(cfg.T, world, K, ms),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.dtype,
        "data": "synthetic",
        "config": {"workload": workload_desc(cfg) + (" +router_gemm" if args.router_gemm else "")
                   + (" +quantize_x" if args.quantize_x else "") + (" +fused_shared" if args.fused_shared else ""),
                   "global_batch": cfg.T * world, "tokens_per_gpu": cfg.T,
                   "parallelism": f"replicas{world}", "l2": l2_note(ab["layer"]), "graph": f"CUDA graphs of {U} steps; the last {U} carry timing events",
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
                       "note": "from the last U steps, whose graph carries timing events"},
        "e2e": {"value": job_tokens_per_s(cfg.T, world, E2E, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": sum(hs.numel() * hs.element_size() for hs in hosts),
                "d2h_bytes_per_step": out_h.numel() * out_h.element_size(), "steps": E2E,
                "api": "StepPipeline.run: per step H2D copies (pinned) -> graph of the step -> D2H copy (pinned), "
                       "the copies of steps i+1 and i-1 overlapping step i on a copy stream",
                "eager": {"value": job_tokens_per_s(cfg.T, world, E2E, eager_ms),
                          "api": "layer.forward() per step (eager C-ABI calls), the same copies serialised with it"}},
        "gpu_launches": K * layer.launches_per_step,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, inp, min_s=10.0, max_s=30.0)
    if rank == 0:
        print(json.dumps(result), flush=True)
    del g_u, g_p, g_1
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------- oracle


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cfg, inp, min_s: float, max_s: float):
    """The CPU oracle, as it stands, on whole steps of the same workload:
    repeated over all T tokens until min_s has passed (at most max_s)."""
    import oracle
    ov = synth.oracle_view(inp)
    c = cfg.as_dict()
    tokens = 0
    t0 = time.time()
    while True:
        oracle.moe_layer(c, ov)
        tokens += cfg.T
        el = time.time() - t0
        if el >= min_s or el + el / max(tokens // cfg.T, 1) > max_s:
            break
    return {"value": tokens / el, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
            "sample": f"{tokens // cfg.T} full step(s) of {cfg.T} tokens, {el:.1f} s (numpy float64; BLAS "
                      f"matrix-vector products threaded, the rest single-threaded)"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    cfg = configs.CONFIGS[args.config]
    inp = synth.oracle_view(synth.make_layer_inputs(cfg))
    c = cfg.as_dict()
    # one unit = one expert MLP of one (token, slot) pair, or one token's shared
    # expert; a token is top_k + 1 units. Steps cycle through the workload.
    cb = inp.get("correction_bias")
    ids, w = oracle.route(c, inp["logits"].numpy(), None if cb is None else cb.numpy())
    mx = cfg.dtype in ("mxfp8", "mxfp4")
    afmt = "mxfp8" if mx else cfg.dtype  # activations and h (MXFP4 layers: MXFP8)
    x = oracle.decode_operand(inp["x"], afmt, inp["x_scale"] if mx else None)
    s_x = inp["x_scale"].reshape(-1).double().numpy() if cfg.dtype == "fp8" else None
    units = [(t, j) for t in range(cfg.T) for j in range(-1, cfg.top_k)]

    def wts(name, e=None):
        """Decoded weights and the fp8 per-matrix scale (1 otherwise)."""
        t, sc = inp[name], inp.get(name + "_scale")
        if e is not None:
            t = t[e]
        if mx:
            return oracle.decode_operand(t, cfg.dtype, sc if e is None else sc[e]), 1.0
        if cfg.dtype == "fp8":
            return oracle.decode_operand(t, "fp8"), float(sc.reshape(-1)[0 if e is None else e])
        return oracle.decode_operand(t, cfg.dtype), 1.0

    def step(i):
        t, j = units[i % len(units)]
        sx = 1.0 if s_x is None else float(s_x[t])
        if j < 0:
            (w13, s13), (w2, s2), inter = wts("w13s"), wts("w2s"), cfg.Is
        else:
            e = ids[t, j]
            (w13, s13), (w2, s2), inter = wts("w13", e), wts("w2", e), cfg.I
        oracle.expert_forward(x[t], w13, w2, inter, afmt, sx, s13, s2)

    for i in range(args.warmup):
        step(i)
    t0 = time.time()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.time() - t0
    tok = args.steps / (cfg.top_k + 1)
    val = tok / el
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(cfg), "global_batch": cfg.T, "parallelism": "cpu"},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
                         "sample": f"each step = one expert MLP of one (token, slot) pair or one shared expert "
                                   f"({cfg.top_k + 1} units = 1 token); {args.steps} units"},
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
