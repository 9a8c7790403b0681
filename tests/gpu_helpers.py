"""Shared helpers of the GPU parity tests: run the C-ABI path on seeded inputs
and compare with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from routed_shared_experts_b200 import capi, synth
from routed_shared_experts_b200.layer import MoELayer

BF16_TOL = 1e-2  # max|out - ref| <= 1e-2 * rms(ref)
FP8_TOL = 3e-2


def to_dev(inp: dict, dev="cuda") -> dict:
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def run_layer(cfg, inp_dev: dict, block_m=None, steps=1):
    layer = MoELayer(cfg, inp_dev, block_m=block_m)
    for _ in range(steps):
        layer.forward()
    torch.cuda.synchronize()
    assert capi.device_error() == 0
    return layer


def oracle_layer(cfg, inp_cpu: dict, tokens=None):
    return oracle.moe_layer(cfg.as_dict(), synth.oracle_view(inp_cpu), tokens=tokens)


def assert_close_rms(out, ref, tol, what=""):
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    ok, err, rms = oracle.tolerance_ok(out, ref, tol)
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    assert ok, f"{what}: max|err| {err:.3e} > {tol} * rms {rms:.3e}"
    return err / max(rms, 1e-30)
