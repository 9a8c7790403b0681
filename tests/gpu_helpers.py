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


def check_routing(cfg, logits, bias, gpu_ids, gpu_w):
    """Routing ids bit-exact against the oracle, weights to 1e-6 relative.

    Grouped sigmoid routing: a token holding a score within the hazard margin
    of an fp32 rounding midpoint (oracle.sigmoid_fp32_hazard_mask) may take the
    other rounding of that score; such a token must then equal the oracle's
    routing evaluated with the other rounding. Returns the tokens whose routing
    equals the oracle's primary one (those the output is compared on)."""
    logits = np.asarray(logits, np.float32)
    ids, w = oracle.route(cfg.as_dict(), logits, bias)
    same = np.all(gpu_ids == ids, axis=1)
    if cfg.route == "grouped_sigmoid":
        mask = oracle.sigmoid_fp32_hazard_mask(logits)
        haz = mask.any(axis=1)
        alt_s = np.where(mask, oracle.sigmoid_fp32_other(logits), oracle.sigmoid_fp32(logits))
        alt_ids, alt_w = oracle.router_grouped_sigmoid_topk(logits, bias, cfg.top_k, cfg.n_group, cfg.topk_group,
                                                            cfg.renormalize, cfg.rsf, scores=alt_s)
        alt = haz & np.all(gpu_ids == alt_ids, axis=1)
        assert np.all(same | alt), f"routing differs at tokens {np.nonzero(~(same | alt))[0][:10]}"
        w = np.where(same[:, None], w, alt_w)
    else:
        assert np.all(same), f"routing differs at tokens {np.nonzero(~same)[0][:10]}"
    np.testing.assert_allclose(gpu_w, w, rtol=1e-6)
    return np.nonzero(same)[0]


def oracle_layer(cfg, inp_cpu: dict, tokens=None):
    return oracle.moe_layer(cfg.as_dict(), synth.oracle_view(inp_cpu), tokens=tokens)


def bf16_ulp(v):
    """Spacing of bf16 numbers at |v| (normal range)."""
    v = np.abs(np.asarray(v, np.float64))
    _, e = np.frexp(np.maximum(v, 2.0**-126))
    return np.ldexp(1.0, (e - 1 - 7).astype(np.int32))


def assert_close_rms(out, ref, tol, what="", rounded=None, exact_frac=None, mean_check=True):
    """Tolerance of the layer's float outputs.

    The stated bound max|out - ref| <= tol * rms(ref) applies to the arithmetic.
    Both sides round the stored results to bf16, and two correct roundings of
    values that differ only in their last fp32 bits can land one bf16 step
    apart, so each element may also differ by one bf16 ulp of every rounded
    quantity listed in ``rounded`` (default: ``ref`` itself). Two checks guard
    against errors hiding in that allowance: mean|err| <= tol/10 * rms(ref)
    (skipped with ``mean_check=False`` where ``ref`` itself carries an extra
    rounding by construction) and,
    when ``exact_frac`` is given, at least that fraction of the elements equal
    the oracle's bit for bit.
    Returns max|err| / rms(ref).
    """
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = np.abs(out - ref)
    terms = [ref] if rounded is None else rounded
    bound = tol * rms + sum(bf16_ulp(t) for t in terms)
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond tol*rms + rounding; worst err "
                           f"{err.max():.3e}, rms {rms:.3e}")
    if mean_check:
        assert err.mean() <= 0.1 * tol * rms, f"{what}: mean|err| {err.mean():.3e} vs rms {rms:.3e}"
    if exact_frac is not None:
        frac = float(np.mean(out == ref))
        assert frac >= exact_frac, f"{what}: only {frac:.3f} of the outputs bit-identical"
    return float(err.max() / max(rms, 1e-30))
