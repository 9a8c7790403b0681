"""Parity of the fp8 a8w8 layer (per-token activation scales, per-expert weight
scales, biased grouped sigmoid routing with the scale folded in, per-row e4m3
quantisation of the stage-1 output) with the CPU oracle.

Tolerance: max|out - ref| <= 3e-2 * rms(ref) plus one bf16 step of each rounded
quantity (see gpu_helpers.assert_close_rms); routing and sort bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import quantised_layer_allowance, stratified_tokens, FP8_TOL, assert_close_rms, check_routing, run_layer
from routed_shared_experts_b200 import configs, synth

pytestmark = pytest.mark.gpu

# several weight tiles in both stages, ragged token blocks, 4 groups of 4 experts
SMALL_FP8 = configs.small(configs.FP8_A8W8, name="small_fp8", T=100, H=512, E=16, top_k=4, I=256, Is=384,
                          n_group=4, topk_group=2, block_m=32, seed=21)


def _check(cfg, tokens=None, block_m=None, device="cuda"):
    inp = synth.make_layer_inputs(cfg, device=device)
    layer = run_layer(cfg, inp if device == "cuda" else {k: (v.cuda() if isinstance(v, torch.Tensor) else v)
                                                          for k, v in inp.items()}, block_m=block_m)
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
    tokens = tokens[np.isin(tokens, agree)]  # tokens routed exactly as the oracle routes them
    ref = oracle.moe_layer(cfg.as_dict(), cpu, tokens=tokens, want_h=True)
    # h codes taken at rounding ties (checked to be ties) and their exact effect
    allow_out, allow_add, _ = quantised_layer_allowance(cfg, layer, cpu, tokens, ref)
    add = layer.addend.float().cpu().numpy()[tokens]
    assert_close_rms(add, ref["addend"], FP8_TOL, "addend", allow=allow_add, exact_frac=0.95)
    out = layer.out.float().cpu().numpy()[tokens]
    rel = assert_close_rms(out, ref["out"], FP8_TOL, "out", rounded=[ref["out"], ref["addend"]],
                         allow=allow_out, exact_frac=0.95)
    assert torch.count_nonzero(layer.acc_ws).item() == 0
    return rel


@pytest.mark.parametrize("block_m", [16, 32, 64, 128])
def test_layer_fp8_small(cuda_lib, block_m):
    _check(SMALL_FP8, block_m=block_m, device="cpu")


def test_layer_fp8_a8w8(cuda_lib):
    """The full fp8 a8w8 layer on a stratified set of >= 256 tokens (one per
    active expert, the hottest expert's ragged last block, blocks spread over
    the GEMMs' waves); routing and sort on every token."""
    _check(configs.FP8_A8W8, tokens="stratified")


@pytest.mark.parametrize("T", configs.SWEEP_T)
def test_layer_fp8_decode_sweep(cuda_lib, T):
    cfg = configs.fp8_decode(T)
    tokens = np.arange(T) if T <= 4 else np.linspace(0, T - 1, 4).astype(int)
    _check(cfg, tokens=tokens)


def test_fp8_stage1_rows_are_scaled_e4m3(cuda_lib):
    """Every stored row of h decodes to values within the e4m3 range, and the
    row's largest code is (close to) 448: the scale is amax/448 per row."""
    cfg = SMALL_FP8
    inp = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in synth.make_layer_inputs(cfg).items()}
    layer = run_layer(cfg, inp)
    n = int(layer.num_padded.item())
    s = layer.sorted_ids.cpu().numpy()[:n]
    valid = s < cfg.T * cfg.top_k
    codes = layer.h.cpu().numpy()[:n][valid]
    vals = np.abs(oracle.e4m3_decode(codes))
    assert np.all(np.isfinite(vals)) and vals.max() <= 448
    assert np.all(vals.max(axis=1) >= 416)  # amax maps to 448 (one e4m3 step below at most)
    assert np.all(layer.h_scale.cpu().numpy()[:n][valid] > 0)
