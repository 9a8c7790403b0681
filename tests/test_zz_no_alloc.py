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

from gpu_helpers import BF16_TOL, assert_close_rms, to_dev
from routed_shared_experts_b200 import capi, configs, synth
from routed_shared_experts_b200.layer import MoELayer

pytestmark = pytest.mark.gpu

MULTI = configs.small(configs.DECODE_BF16, name="multi_bf16", T=53, H=384, E=16, top_k=4, I=192, Is=128,
                      seed=11)


def _static_stage2(layer, out):
    cfg, inp = layer.cfg, layer.inp
    capi.moe_stage2_gemm_accumulate_static_ws(
        layer.dt, layer.h, layer.h_scale, inp["w2"], layer.wsc["w2"], layer.topk_weights, capi.MOE_DT_F32,
        layer.sorted_ids, layer.block_expert, layer.num_padded, cfg.T, cfg.top_k, cfg.H, cfg.I, cfg.E, layer.bm,
        layer.addend, None, out)


@pytest.mark.parametrize("cfg", [MULTI, configs.DECODE_BF16], ids=lambda c: c.name)
def test_static_workspace_matches_caller_workspace(cuda_lib, cfg):
    inp = to_dev(synth.make_layer_inputs(cfg))
    layer = MoELayer(cfg, inp)
    layer.forward()  # routed stage 2 with the caller's workspace, addend from the side stream
    torch.cuda.synchronize()
    ref = layer.out.float().cpu().numpy()
    for call in range(2):  # two calls in a row share the static array
        out = torch.full_like(layer.out, float("nan"))
        _static_stage2(layer, out)
        torch.cuda.synchronize()
        assert capi.device_error() == 0
        assert_close_rms(out.float().cpu().numpy(), ref, BF16_TOL, f"static workspace, call {call}",
                         exact_frac=0.95)


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
