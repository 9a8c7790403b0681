"""The shared expert as always-selected routed experts (FusedSharedMoELayer,
moe_append_shared_slots) against the oracle's fused mode: one launch per
stage for routed and shared experts, all contributions summed before the one
rounding. Shapes cover a shared expert narrower than a routed one (one
zero-padded piece), wider (several pieces), equal, gated and not, bf16, fp8
and MXFP8, small and decode-sized token tiles."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import BF16_TOL, FP8_TOL, assert_close_rms, check_routing
from routed_shared_experts_b200 import capi, configs, synth
from routed_shared_experts_b200.layer import FusedSharedMoELayer

pytestmark = pytest.mark.gpu


def _check(cfg, block_m=None, device="cpu", tokens=None):
    inp = synth.make_layer_inputs(cfg, device=device)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    layer = FusedSharedMoELayer(cfg, dev, block_m=block_m)
    layer.forward()
    torch.cuda.synchronize()
    assert capi.device_error() == 0
    assert torch.count_nonzero(layer.acc_ws).item() == 0
    cpu = synth.oracle_view(inp)
    bias = None if cpu.get("correction_bias") is None else cpu["correction_bias"].numpy()
    agree = check_routing(cfg, cpu["logits"].numpy(), bias, layer.topk_ids.cpu().numpy(),
                          layer.topk_weights.cpu().numpy())
    ids2 = layer.ids2.cpu().numpy()
    assert np.array_equal(ids2[:, : cfg.top_k], layer.topk_ids.cpu().numpy())
    assert np.all(ids2[:, cfg.top_k:] == np.arange(cfg.E, cfg.E + layer.m)[None, :])
    tokens = agree if tokens is None else np.intersect1d(agree, tokens)
    ref = oracle.moe_layer(cfg.as_dict(), cpu, tokens=tokens, shared_fused=True)
    out = layer.out.float().cpu().numpy()[tokens]
    tol = BF16_TOL if cfg.dtype == "bf16" else FP8_TOL
    return assert_close_rms(out, ref["out"], tol, "out", rounded=[ref["out"]])


@pytest.mark.parametrize("Is,block_m", [(128, 16), (320, 16), (256, 64), (128, 128)])
def test_fused_shared_bf16(cuda_lib, Is, block_m):
    cfg = configs.small(configs.DECODE_BF16, name="fs_bf16", T=48, H=512, E=16, top_k=4, I=128, Is=Is, seed=51)
    _check(cfg, block_m=block_m)


def test_fused_shared_bf16_decode_layer(cuda_lib):
    cfg = configs.DECODE_BF16  # Is = 512 < I = 768: one zero-padded piece
    _check(cfg, device="cuda", tokens=np.arange(0, 32, 3))


@pytest.mark.parametrize("block_m", [16, 128])
def test_fused_shared_fp8(cuda_lib, block_m):
    cfg = configs.small(configs.FP8_A8W8, name="fs_fp8", T=100, H=512, E=16, top_k=4, I=256, Is=512,
                        n_group=4, topk_group=2, seed=52)  # Is = 2 I: two pieces with their own row scales
    _check(cfg, block_m=block_m)


def test_fused_shared_mx(cuda_lib):
    cfg = configs.small(configs.MXFP8_PREFILL, name="fs_mx", T=72, H=512, E=8, top_k=2, I=256, Is=256,
                        n_group=4, topk_group=2, block_m=32, seed=53)
    _check(cfg)
