"""Run a few layer forwards of one workload, for profiler captures.

    python -m routed_shared_experts_b200.profile_step [--config decode_bf16]
        [--warmup 2] [--routed-only] [--tokens T] [--experts E]

Builds the workload's seeded inputs on cuda:0, runs ``--warmup`` full layer
forwards, then one more forward (or only the routed half with
``--routed-only``), synchronises and checks the device error word. Nothing is
timed here; it exists so that a profiler can be pointed at a known, short
sequence of launches. ``--tokens`` / ``--experts`` shrink the workload (same
shapes otherwise) for captures that must stay within a few GB of device memory.
"""
from __future__ import annotations

import argparse

import torch

from . import capi, configs, synth
from .layer import MoELayer


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="decode_bf16")
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--routed-only", action="store_true")
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--experts", type=int, default=None)
    a = ap.parse_args()
    cfg = configs.CONFIGS[a.config]
    over = {}
    if a.tokens:
        over["T"] = a.tokens
    if a.experts:
        over["E"] = a.experts
    if over:
        cfg = configs.small(cfg, name=cfg.name + "_reduced", **over)
    inp = synth.make_layer_inputs(cfg, device="cuda")
    layer = MoELayer(cfg, inp)
    for _ in range(a.warmup):
        layer.forward()
    if a.routed_only:
        layer.routed(torch.cuda.current_stream(), addend=False)
    else:
        layer.forward()
    torch.cuda.synchronize()
    code = capi.device_error()
    if code:
        raise SystemExit(f"device error {code}")
    print("ok", cfg.name, "active experts", int((layer.expert_counts > 0).sum()))


if __name__ == "__main__":
    main()
