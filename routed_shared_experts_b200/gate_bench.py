"""Latency of the fused shared-expert gate, sigmoid(x . w_gate), for one token.

    python -m routed_shared_experts_b200.gate_bench [--reps 2000]

For K in {1024, 2048, 4096} and bf16 / fp16 inputs (x ~ N(0,1), w ~ N(0,0.02),
seeded), prints one JSON line per case: the time per call replayed from a CUDA
graph of `reps` back-to-back calls (launch included, as in a decode step), the
same for a near-empty kernel (the launch floor on this GPU), and the bytes the
call must read. The pages' context for this microbenchmark is vllm-project/vllm
PR 56789, "Kernel microbenchmark" (one token, K = 2048, on another GPU).
"""
from __future__ import annotations

import argparse
import json

import torch

from . import capi, configs, synth


def _graph_us(fn, reps: int, stream) -> float:
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                fn()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(5):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / (5 * reps)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--reps", type=int, default=2000)
    a = ap.parse_args()
    s = torch.cuda.Stream()
    floor = _graph_us(lambda: torch.cuda._sleep(0), a.reps, s)
    for dt in configs.GATE_DTYPES:
        for K in configs.GATE_K:
            x, w = synth.make_gate_inputs(K, dt, configs.GATE_SEED, T=1, device="cuda")
            out = torch.empty(1, dtype=x.dtype, device="cuda")
            code = capi.MOE_DT_BF16 if dt == "bf16" else capi.MOE_DT_FP16
            us = _graph_us(lambda: capi.shared_expert_gate_dot(code, x, w, True, out, s), a.reps, s)
            print(json.dumps({"workload": f"shared_expert_gate T=1 K={K} {dt}", "us_per_call": us,
                              "launch_floor_us": floor, "bytes": 2 * K * 2 + 2,
                              "timing": f"CUDA graph of {a.reps} calls"}), flush=True)


if __name__ == "__main__":
    main()
