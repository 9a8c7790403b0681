"""moe_quantize_activations: bf16 activations to the fp8 (per-token scale)
and MXFP8 (ue8m0 per 32 columns) stage-1 formats, bit-exact against the
oracle's codes and scales, and a layer that starts from bf16 x."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import FP8_TOL, assert_close_rms, check_routing
from routed_shared_experts_b200 import capi, configs, synth
from routed_shared_experts_b200.layer import MoELayer

pytestmark = pytest.mark.gpu


def _x(T, H, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, generator=g)
    if T > 2:
        x[1] = 0                      # an all-zero row
        x[2, 5] = 300.0               # one outlier
        x[2, 40:72] = 0               # an all-zero MX block (when 32-aligned)
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("T,H", [(1, 4096), (37, 2048), (16, 7168), (9, 256), (3, 8)])
def test_quantize_fp8_bit_exact(cuda_lib, T, H):
    x = _x(T, H, seed=T + H)
    q = torch.empty(T, H, dtype=torch.uint8, device="cuda")
    s = torch.empty(T, dtype=torch.float32, device="cuda")
    capi.moe_quantize_activations(capi.MOE_DT_FP8_E4M3, x.cuda(), q, s)
    torch.cuda.synchronize()
    rc, rs = oracle.quantize_activations(x.double().numpy(), "fp8")
    assert np.array_equal(q.cpu().numpy(), rc)
    assert np.array_equal(s.cpu().numpy(), rs)


@pytest.mark.parametrize("T,H", [(1, 4096), (37, 2048), (16, 7168), (9, 96)])
def test_quantize_mx_bit_exact(cuda_lib, T, H):
    x = _x(T, H, seed=3 * T + H)
    q = torch.empty(T, H, dtype=torch.uint8, device="cuda")
    sb = torch.empty(T, H // 32, dtype=torch.uint8, device="cuda")
    capi.moe_quantize_activations(capi.MOE_DT_MXFP8_E4M3, x.cuda(), q, sb)
    torch.cuda.synchronize()
    rc, rs = oracle.quantize_activations(x.double().numpy(), "mxfp8")
    assert np.array_equal(q.cpu().numpy(), rc)
    assert np.array_equal(sb.cpu().numpy(), rs)


@pytest.mark.parametrize("base", [configs.FP8_A8W8, configs.MXFP8_PREFILL])
def test_layer_from_bf16_activations(cuda_lib, base):
    """The layer quantises its bf16 x in the step; the oracle, fed with its own
    quantisation of the same x, gives the same output within the tolerance."""
    kw = dict(T=64, H=512, E=16, top_k=4, I=256, Is=256, n_group=4, topk_group=2, block_m=32, seed=41)
    cfg = configs.small(base, name="qx_" + base.dtype, **kw)
    inp = synth.make_layer_inputs(cfg)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    layer = MoELayer(cfg, dev, quantize_x=True)
    layer.forward()
    torch.cuda.synchronize()
    assert capi.device_error() == 0
    codes, scale = oracle.quantize_activations(inp["x_r"].double().numpy(), cfg.dtype)
    assert np.array_equal(layer.xq.cpu().numpy(), codes)
    assert np.array_equal(layer.xq_scale.cpu().numpy(), scale)
    cpu = dict(synth.oracle_view(inp), x=torch.from_numpy(codes), x_scale=torch.from_numpy(scale))
    bias = None if cpu.get("correction_bias") is None else cpu["correction_bias"].numpy()
    agree = check_routing(cfg, cpu["logits"].numpy(), bias, layer.topk_ids.cpu().numpy(),
                          layer.topk_weights.cpu().numpy())
    ref = oracle.moe_layer(cfg.as_dict(), cpu, tokens=agree)
    out = layer.out.float().cpu().numpy()[agree]
    assert_close_rms(out, ref["out"], FP8_TOL, "out", rounded=[ref["out"], ref["addend"]])
