"""Stage 2 with the library's static workspace (moe_stage2_gemm_accumulate_static_ws).

That entry point serves callers that cannot allocate device memory (operator
plugin interfaces that receive only input and output buffers, or processes
whose device memory already belongs to another allocator's pool). It must give
the same output as moe_stage2_gemm_accumulate with a caller-provided
workspace, call after call, since every call reuses the same static array.

This file is collected last on purpose and also passes when run alone in a
fresh process (the static array starts zeroed and each call clears what it
uses).
"""
import pytest
import torch

from gpu_helpers import BF16_TOL, FP8_TOL, assert_close_rms, to_dev
from routed_shared_experts_b200 import capi, configs, synth
from routed_shared_experts_b200.layer import MoELayer

pytestmark = pytest.mark.gpu

MULTI = configs.small(configs.DECODE_BF16, name="multi_bf16", T=53, H=384, E=16, top_k=4, I=192, Is=128,
                      seed=11)
SMALL_FP8 = configs.small(configs.FP8_A8W8, name="noalloc_fp8", T=60, H=512, E=16, top_k=4, I=256, Is=256,
                          n_group=4, topk_group=2, block_m=32, seed=41)
# 128-token blocks with an even number of weight tiles: stage 2 on CTA pairs
SMALL_MX = configs.small(configs.MXFP8_PREFILL, name="noalloc_mx", T=150, H=512, E=8, top_k=2, I=256, Is=256,
                         n_group=4, topk_group=2, block_m=128, seed=42)


def _static_stage2(layer, out):
    cfg, inp = layer.cfg, layer.inp
    capi.moe_stage2_gemm_accumulate_static_ws(
        layer.dt, layer.h, layer.h_scale, inp["w2"], layer.wsc["w2"], layer.topk_weights, capi.MOE_DT_F32,
        layer.sorted_ids, layer.block_expert, layer.num_padded, cfg.T, cfg.top_k, cfg.H, cfg.I, cfg.E, layer.bm,
        layer.addend, None, out)


@pytest.mark.parametrize("cfg", [MULTI, configs.DECODE_BF16, SMALL_FP8, SMALL_MX], ids=lambda c: c.name)
def test_static_workspace_matches_caller_workspace(cuda_lib, cfg):
    inp = to_dev(synth.make_layer_inputs(cfg))
    layer = MoELayer(cfg, inp)
    layer.forward()  # routed stage 2 with the caller's workspace, addend from the side stream
    torch.cuda.synchronize()
    ref = layer.out.float().cpu().numpy()
    tol = BF16_TOL if cfg.dtype == "bf16" else FP8_TOL
    for call in range(2):  # two calls in a row share the static array
        out = torch.full_like(layer.out, float("nan"))
        _static_stage2(layer, out)
        torch.cuda.synchronize()
        assert capi.device_error() == 0
        assert_close_rms(out.float().cpu().numpy(), ref, tol, f"static workspace, call {call}", exact_frac=0.95)


def test_static_workspace_call_allocates_nothing(cuda_lib):
    """A warmed-up call changes neither the caching allocator's allocation
    count nor the device's free memory (no cudaMalloc behind the caller's
    back)."""
    cfg = MULTI
    inp = to_dev(synth.make_layer_inputs(cfg))
    layer = MoELayer(cfg, inp)
    layer.forward()
    out = torch.empty_like(layer.out)
    _static_stage2(layer, out)  # first call: looks up the array's address, loads the kernel
    torch.cuda.synchronize()
    n0 = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        _static_stage2(layer, out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_stats().get("allocation.all.allocated", 0) == n0
    assert free1 == free0
    assert capi.device_error() == 0


def test_static_workspace_rejects_oversized_problem(cuda_lib):
    T, H = 4096, 2048  # needs 32 MiB + counters
    assert capi.stage2_workspace_bytes(T, H) > 8 << 20
    dummy = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(capi.MoEError) as ei:
        capi.moe_stage2_gemm_accumulate_static_ws(capi.MOE_DT_BF16, dummy, None, dummy, None, None,
                                                  capi.MOE_DT_F32, ids, ids, ids, T, 8, H, 768, 128, 16, None,
                                                  None, dummy)
    assert ei.value.status == -7
