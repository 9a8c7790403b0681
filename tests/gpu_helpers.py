"""Shared helpers of the GPU parity tests: run the C-ABI path on seeded inputs
and compare with the CPU oracle."""
from __future__ import annotations

import json
import os

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


def stratified_tokens(cfg, topk_ids, block_m=None, n_min=256, seed=0):
    """Tokens to compare on a layer too large to check whole: at least one
    token of every active expert, every token of the hottest expert's last
    (ragged) token block, the first token of blocks spread over the whole
    sorted order (so blocks that run in different waves of the persistent
    GEMMs are covered), then seeded random tokens up to n_min."""
    ids = np.asarray(topk_ids)
    k, bm = cfg.top_k, block_m or cfg.block_m
    srt = oracle.align_sort(ids, cfg.E, bm)
    s, off, cnt = srt["sorted_ids"], srt["expert_offsets"], srt["expert_counts"]
    sel = set()
    for e in np.nonzero(cnt)[0]:
        sel.add(int(s[off[e]]) // k)
    hot = int(np.argmax(cnt))
    last0 = off[hot] + (int(cnt[hot]) - 1) // bm * bm
    for r in range(last0, off[hot] + int(cnt[hot])):
        sel.add(int(s[r]) // k)
    nblk = len(srt["block_expert"])
    for b in range(0, nblk, max(1, nblk // 64)):
        f = int(s[b * bm])
        if f < cfg.T * k:
            sel.add(f // k)
    rng = np.random.default_rng(seed)
    rest = [t for t in rng.permutation(cfg.T) if t not in sel]
    sel.update(int(t) for t in rest[: max(0, n_min - len(sel))])
    return np.array(sorted(sel))


def _report(rec):
    """Appends one parity record (JSON line) to $PARITY_REPORT, if set."""
    path = os.environ.get("PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


def assert_close_rms(out, ref, tol, what="", rounded=None, exact_frac=None, mean_check=True, allow=None):
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
    if allow is not None:  # the exact effect of h codes taken at rounding ties (quantised layers)
        bound = bound + allow
    bad = err > bound
    # the literal stated bound, reported beside the checked one
    import inspect
    caller = next((f.function for f in inspect.stack()[1:] if f.function.startswith("test_")), "?")
    _report({"test": os.environ.get("PYTEST_CURRENT_TEST", caller).split(" ")[0], "what": what, "tol": tol,
             "n": int(err.size), "max_err_over_rms": float(err.max() / max(rms, 1e-30)) if err.size else 0.0,
             "mean_err_over_rms": float(err.mean() / max(rms, 1e-30)) if err.size else 0.0,
             "beyond_tol_rms": int(np.sum(err > tol * rms)), "exact_frac": float(np.mean(out == ref)),
             "exact_frac_guard": exact_frac,
             "elements_with_tie_allowance": 0 if allow is None else int(np.sum(np.broadcast_to(allow, err.shape) > 0)),
             "beyond_tol_rms_without_tie_allowance": int(np.sum((err > tol * rms) & (
                 np.broadcast_to(allow, err.shape) == 0))) if allow is not None else int(np.sum(err > tol * rms))})
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond tol*rms + rounding; worst err "
                           f"{err.max():.3e}, rms {rms:.3e}")
    if mean_check:
        assert err.mean() <= 0.1 * tol * rms, f"{what}: mean|err| {err.mean():.3e} vs rms {rms:.3e}"
    if exact_frac is not None:
        frac = float(np.mean(out == ref))
        assert frac >= exact_frac, f"{what}: only {frac:.3f} of the outputs bit-identical"
    return float(err.max() / max(rms, 1e-30))


# ---------------------------------------------------------------------------
# Quantised layers: the stage-1 output h is re-quantised on each side (the GPU
# from its fp32 h, the oracle from its float64 h). Where a value sits at a
# rounding tie of e4m3 (or an MX block's amax at a power of two), both codes
# are correct results of the layer's arithmetic; the two sides may then take
# different codes and their outputs differ by exactly that code difference
# times the W2 column. The helpers below find the codes the GPU took that
# differ from the oracle's, check that each one is such a tie, and bound the
# outputs' difference by the exact effect of those codes.
# ---------------------------------------------------------------------------

HFLIP_MARGIN = 2.0 ** -12  # relative distance to a tie within which both roundings are accepted


def _e4m3_values(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn)
    return t.double().numpy()


def gpu_h_values(layer, rows, shared=False):
    """float64 values of the GPU's stored stage-1 rows (sorted-order rows of
    ``layer.h``, or rows of the shared expert's ``layer.h_s``), decoded from
    the formats the library documents: bf16; e4m3 codes times the row's fp32
    scale; e4m3 codes times 2^(b - 127) with the ue8m0 bytes read from the
    512-byte scale tiles (byte (r % 32) * 16 + (r / 32) * 4 + (b % 4) of tile
    (row block, b / 4))."""
    cfg = layer.cfg
    h = (layer.h_s if shared else layer.h)[torch.as_tensor(rows, device=layer.h.device)]
    if cfg.dtype == "bf16":
        return h.double().cpu().numpy()
    codes = h.cpu().numpy()
    vals = _e4m3_values(codes)
    sc = layer.h_scale_s if shared else layer.h_scale
    if cfg.dtype == "fp8":
        # the e4m3 values of the codes (the GPU's row scale, continuous, is returned apart)
        return vals, sc.cpu().numpy()[rows].astype(np.float64)
    ncol = codes.shape[1]
    bm = layer.bm
    rr = np.asarray(rows) % bm
    blk = np.asarray(rows) // bm
    b = np.arange(ncol // 32)
    off = ((blk[:, None] * (ncol // 128) + b[None, :] // 4) * 512 + (rr[:, None] % 32) * 16
           + (rr[:, None] // 32) * 4 + (b[None, :] % 4))
    sb = sc.cpu().numpy()[off].astype(np.int64)
    return vals * np.repeat(np.ldexp(1.0, (sb - 127).astype(np.int32)), 32, axis=1)


def _tie_distance(a):
    """Distance of |a| (e4m3-scaled values, < 448) to the nearest rounding
    midpoint of the e4m3 grid: steps 2^(e-3) in binade e >= -6, 2^-9 below."""
    a = np.abs(a)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    step = np.ldexp(1.0, (e - 3).astype(np.int32))
    mid = (np.floor(a / step) + 0.5) * step
    return np.abs(a - mid), step


def h_flip_check(cfg, h_gpu, h_raw, h_q):
    """Codes of the GPU's h [..., n] that differ from the oracle's h_q, each
    checked to be the other rounding of a tie of the oracle's unquantised
    h_raw; returns the value difference those codes make, |dh| (zero where the
    codes agree). fp8: h_gpu is (e4m3 values of the codes, the GPU's row
    scales); the per-row scale amax/448 is continuous and may differ from the
    oracle's in its last bit, which scales a whole row by about 1e-7 (inside
    the output tolerance), so codes are compared, and a differing code counts
    at the oracle's scale."""
    if cfg.dtype == "fp8":
        q_gpu, _ = h_gpu
        amax = np.max(np.abs(h_raw), axis=-1, keepdims=True)
        s_or = np.where(amax > 0, oracle.fp32_round(amax / 448.0), 1.0)
        d = (q_gpu.reshape(h_q.shape) - h_q / s_or) * s_or
    else:
        d = h_gpu - h_q
    flips = d != 0
    if not flips.any():
        return np.zeros_like(d)
    assert flips.sum() <= max(8, 1e-3 * flips.size), f"{flips.sum()} of {flips.size} h codes differ from the oracle's"
    n = h_raw.shape[-1]
    if cfg.dtype == "fp8":
        amax = np.max(np.abs(h_raw), axis=-1, keepdims=True)
        s = np.where(amax > 0, oracle.fp32_round(amax / 448.0), 1.0)
        v = h_raw / s
        dist, step = _tie_distance(v)
        ok = dist <= HFLIP_MARGIN * np.maximum(np.abs(v), 1.0)
        bound = step * s * (1 + 1e-5)
    else:  # MXFP8 h (also the MXFP4 layers' h)
        blk = h_raw.reshape(h_raw.shape[:-1] + (n // 32, 32))
        amax = np.max(np.abs(blk), axis=-1, keepdims=True)
        X = oracle.mx_block_exponent(amax).astype(np.float64)
        v = blk / np.ldexp(1.0, X.astype(np.int32))
        dist, step = _tie_distance(v)
        near_pow2 = np.abs(np.log2(np.maximum(amax, 1e-300)) - np.round(np.log2(np.maximum(amax, 1e-300)))) \
            <= HFLIP_MARGIN / np.log(2)
        elem = dist <= HFLIP_MARGIN * np.maximum(np.abs(v), 1.0)
        ok = (elem | near_pow2).reshape(h_raw.shape)
        # one code step; a different block exponent re-quantises the block: within a quarter of
        # the value plus one subnormal step at the larger exponent
        b_elem = (step * np.ldexp(1.0, X.astype(np.int32))).reshape(h_raw.shape)
        b_exp = (0.25 * np.abs(blk) + np.ldexp(1.0, (X + 1 - 9).astype(np.int32))).reshape(h_raw.shape)
        bound = np.where(np.broadcast_to(near_pow2, blk.shape).reshape(h_raw.shape), np.maximum(b_elem, b_exp), b_elem)
        bound = bound * (1 + 1e-5)
    bad = flips & ~ok
    assert not bad.any(), f"{bad.sum()} h codes differ from the oracle's away from a rounding tie"
    big = flips & (np.abs(d) > bound)
    assert not big.any(), f"{big.sum()} h codes differ from the oracle's by more than a tie allows"
    return np.abs(d)


def quantised_layer_allowance(cfg, layer, inp, tokens, ref):
    """Per-output allowance [n, H] for the h codes the GPU took differently from
    the oracle (each checked to be a tie): sum over the differing codes of
    |top-k weight * W2 scale * W2[n, i] * dh_i| for the routed slots, and the
    same with the gate for the shared expert (and its addend). Returns
    (allow_out, allow_addend, flip count)."""
    T, H, k, I, Is = cfg.T, cfg.H, cfg.top_k, cfg.I, cfg.Is
    srt = layer.sorted_ids.cpu().numpy()[: int(layer.num_padded.item())]
    row_of = np.full(T * k, -1)
    valid = srt < T * k
    row_of[srt[valid]] = np.nonzero(valid)[0]
    slots = (np.asarray(tokens)[:, None] * k + np.arange(k)[None, :]).reshape(-1)
    rows = row_of[slots]
    assert np.all(rows >= 0)
    hg = gpu_h_values(layer, rows)
    hg = (hg[0].reshape(len(tokens), k, I), hg[1]) if cfg.dtype == "fp8" else hg.reshape(len(tokens), k, I)
    d_r = h_flip_check(cfg, hg, ref["h_raw"], ref["h_q"])
    hs = gpu_h_values(layer, np.asarray(tokens), shared=True)
    d_s = h_flip_check(cfg, hs, ref["h_raw_shared"], ref["h_q_shared"])
    fmt = cfg.dtype
    ids = ref["topk_ids"]
    wts = ref["topk_weights"]
    allow_out = np.zeros((len(tokens), H))
    allow_add = np.zeros((len(tokens), H))
    cache = {}

    def w2_of(e):
        if e not in cache:
            if e < 0:
                w, sc = inp["w2s"], inp.get("w2s_scale")
            else:
                w, sc = inp["w2"][e], (inp["w2_scale"][e] if inp.get("w2_scale") is not None else None)
            if fmt == "fp8":
                cache[e] = oracle.decode_operand(w, "fp8") * float(np.asarray(sc.cpu() if torch.is_tensor(sc) else sc).reshape(-1)[0])
            else:
                cache[e] = oracle.decode_operand(w, fmt, sc)
        return cache[e]
    for i, t in enumerate(tokens):
        for j in range(k):
            nz = np.nonzero(d_r[i, j])[0]
            if len(nz):
                allow_out[i] += abs(wts[t, j]) * (np.abs(w2_of(int(ids[t, j]))[:, nz]) @ d_r[i, j, nz])
        nz = np.nonzero(d_s[i])[0]
        if len(nz):
            a = abs(ref["gate"][i]) * (np.abs(w2_of(-1)[:, nz]) @ d_s[i, nz])
            allow_add[i] += a
            allow_out[i] += a
    return allow_out, allow_add, int((d_r != 0).sum() + (d_s != 0).sum())
