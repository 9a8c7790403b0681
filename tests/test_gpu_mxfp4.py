"""Parity of the MXFP4-weight layer (e2m1 weights two per byte with one ue8m0
scale per 32 K elements, MXFP8 activations and h, block-scaled tensor-core MMA
with A declared e2m1) with the CPU oracle.

Beyond the MXFP8 cases (structured scale patterns, every token tile, a hidden
size that is not a multiple of 512, the full prefill layer on sampled tokens)
two cases isolate the 4-bit storage: weights whose even (or odd) elements are
all zero fail if the two codes of a byte were taken in the other order, and a
layer whose weights all carry code 0b0111 (6.0) checks the decoded magnitude.
Tolerance: 3e-2 * rms(ref) plus one bf16 step of each rounded quantity;
routing and sort bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import quantised_layer_allowance, stratified_tokens, FP8_TOL, assert_close_rms, check_routing, run_layer
from routed_shared_experts_b200 import capi, configs, synth
from routed_shared_experts_b200.layer import FusedSharedMoELayer

pytestmark = pytest.mark.gpu

SMALL_MX4 = configs.small(configs.MXFP4_PREFILL, name="small_mx4", T=72, H=512, E=8, top_k=2, I=256, Is=256,
                          n_group=4, topk_group=2, block_m=32, seed=41)
WEIGHTS = ("w13", "w2", "w13s", "w2s")


def _pattern(shape, kind, rng):
    """ue8m0 bytes of the given shape [..., rows, K/32]."""
    if kind == "const":
        return np.full(shape, 124, np.uint8)
    if kind == "rows":
        v = rng.integers(118, 130, shape[:-1] + (1,))
        return np.broadcast_to(v, shape).astype(np.uint8)
    if kind == "kblocks":
        v = rng.integers(118, 130, (1,) * (len(shape) - 1) + (shape[-1],))
        return np.broadcast_to(v, shape).astype(np.uint8)
    raise ValueError(kind)


def _inputs(cfg, wpat=None, codes=None, seed=0):
    inp = synth.make_layer_inputs(cfg)
    rng = np.random.default_rng(seed)
    if wpat:
        for k in WEIGHTS:
            inp[k + "_scale"] = torch.from_numpy(_pattern(tuple(inp[k + "_scale"].shape), wpat, rng).copy())
    if codes == "even_zero":    # element 2j zero: only the high nibbles carry codes
        for k in WEIGHTS:
            inp[k] = inp[k] & 0xF0
    elif codes == "odd_zero":   # element 2j+1 zero: only the low nibbles
        for k in WEIGHTS:
            inp[k] = inp[k] & 0x0F
    elif codes == "all_six":    # every element 6.0 (0b0111), half of them negated by the byte's sign pattern
        for k in WEIGHTS:
            inp[k] = torch.where(inp[k] < 128, torch.full_like(inp[k], 0x77), torch.full_like(inp[k], 0xFF))
    return inp


def _check(cfg, inp, tokens=None, block_m=None):
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    layer = run_layer(cfg, dev, block_m=block_m)
    cpu = synth.oracle_view(inp)
    bias = None if cpu.get("correction_bias") is None else cpu["correction_bias"].numpy()
    agree = check_routing(cfg, cpu["logits"].numpy(), bias, layer.topk_ids.cpu().numpy(),
                          layer.topk_weights.cpu().numpy())
    ids = layer.topk_ids.cpu().numpy()
    srt = oracle.align_sort(ids, cfg.E, block_m or cfg.block_m)
    n = int(layer.num_padded.item())
    assert n == srt["num_padded"]
    assert np.array_equal(layer.sorted_ids.cpu().numpy()[:n], srt["sorted_ids"])
    if isinstance(tokens, str):  # "stratified": chosen from the routing the layer took
        tokens = stratified_tokens(cfg, layer.topk_ids.cpu().numpy(), block_m)
    tokens = np.arange(cfg.T) if tokens is None else np.asarray(tokens)
    tokens = tokens[np.isin(tokens, agree)]
    ref = oracle.moe_layer(cfg.as_dict(), cpu, tokens=tokens, want_h=True)
    # h codes taken at rounding ties (checked to be ties) and their exact effect
    allow_out, allow_add, _ = quantised_layer_allowance(cfg, layer, cpu, tokens, ref)
    add = layer.addend.float().cpu().numpy()[tokens]
    assert_close_rms(add, ref["addend"], FP8_TOL, "addend", allow=allow_add, exact_frac=0.95)
    out = layer.out.float().cpu().numpy()[tokens]
    assert np.any(ref["out"] != 0)
    return assert_close_rms(out, ref["out"], FP8_TOL, "out", rounded=[ref["out"], ref["addend"]],
                         allow=allow_out, exact_frac=0.95)


@pytest.mark.parametrize("wpat", ["const", "rows", "kblocks"])
def test_mxfp4_structured_scales(cuda_lib, wpat):
    _check(SMALL_MX4, _inputs(SMALL_MX4, wpat))


@pytest.mark.parametrize("codes", ["even_zero", "odd_zero", "all_six"])
def test_mxfp4_nibble_order_and_magnitude(cuda_lib, codes):
    _check(SMALL_MX4, _inputs(SMALL_MX4, "const", codes))


@pytest.mark.parametrize("block_m", [16, 32, 64, 128])
def test_mxfp4_random(cuda_lib, block_m):
    _check(SMALL_MX4, _inputs(SMALL_MX4), block_m=block_m)


@pytest.mark.parametrize("block_m", [16, 128])
def test_mxfp4_hidden_not_multiple_of_512(cuda_lib, block_m):
    cfg = configs.small(SMALL_MX4, name="small_mx4_h640", H=640, seed=43)
    _check(cfg, _inputs(cfg), block_m=block_m)


def test_mxfp4_decode_layer(cuda_lib):
    cfg = configs.MXFP4_DECODE
    _check(cfg, synth.make_layer_inputs(cfg))


def test_mxfp4_prefill_layer(cuda_lib):
    """The full MXFP4 prefill layer on a stratified set of >= 256 tokens: one
    per active expert, the hottest expert's ragged last block, blocks spread
    over the waves of the persistent GEMMs (routing and sort: every token)."""
    cfg = configs.MXFP4_PREFILL
    inp = synth.make_layer_inputs(cfg, device="cuda")
    _check(cfg, inp, tokens="stratified")


def test_mxfp4_fused_shared(cuda_lib):
    cfg = configs.small(SMALL_MX4, name="small_mx4_fused", Is=384, seed=45)
    inp = synth.make_layer_inputs(cfg)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    layer = FusedSharedMoELayer(cfg, dev)
    layer.forward()
    torch.cuda.synchronize()
    assert capi.device_error() == 0
    cpu = synth.oracle_view(inp)
    bias = None if cpu.get("correction_bias") is None else cpu["correction_bias"].numpy()
    agree = check_routing(cfg, cpu["logits"].numpy(), bias, layer.topk_ids.cpu().numpy(),
                          layer.topk_weights.cpu().numpy())
    ref = oracle.moe_layer(cfg.as_dict(), cpu, tokens=agree, shared_fused=True)
    out = layer.out.float().cpu().numpy()[agree]
    assert_close_rms(out, ref["out"], FP8_TOL, "out", rounded=[ref["out"]])
