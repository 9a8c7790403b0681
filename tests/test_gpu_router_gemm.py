"""Parity of the fused router linear + top-k (moe_router_gemm_topk) with the
CPU oracle.

The logits must equal the oracle's fixed-order fp32 sum (oracle.router_logits)
bit for bit, and the routing taken from them must equal both the oracle's and
that of moe_router_topk fed with the same logits. Shapes cover one and many
lanes per token (E = 8 ... 512), token counts that are not a multiple of the
4-token cluster, H from 256 to 7168, bf16 and fp16, both routing modes."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import check_routing, run_layer, assert_close_rms, BF16_TOL
from routed_shared_experts_b200 import capi, configs, synth

pytestmark = pytest.mark.gpu


def _inputs(T, H, E, dtype, seed, bias_std=0.5):
    g = torch.Generator().manual_seed(seed)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    x = torch.randn(T, H, generator=g).to(tdt)
    w = (torch.randn(H, E, generator=g) * 0.02).to(tdt)
    lb = torch.randn(E, generator=g) * bias_std
    return x, w, lb


def _gpu(x, w, lb, cb, cfg):
    T, E = x.shape[0], w.shape[1]
    dev = dict(device="cuda")
    logits = torch.full((T, E), float("nan"), dtype=torch.float32, **dev)
    ids = torch.empty((T, cfg.top_k), dtype=torch.int32, **dev)
    wts = torch.empty((T, cfg.top_k), dtype=torch.float32, **dev)
    mode = capi.MOE_ROUTE_SOFTMAX if cfg.route == "softmax" else capi.MOE_ROUTE_GROUPED_SIGMOID
    cbd = None if cb is None else cb.cuda()
    capi.moe_router_gemm_topk(x.cuda(), w.cuda(), None if lb is None else lb.cuda(), cbd, cfg.top_k, mode,
                              cfg.n_group, cfg.topk_group, cfg.renormalize, cfg.rsf, logits, ids, wts)
    # the logits-input router on the same logits
    ids2 = torch.empty_like(ids)
    wts2 = torch.empty_like(wts)
    capi.moe_router_topk(logits, cbd, cfg.top_k, mode, cfg.n_group, cfg.topk_group, cfg.renormalize, cfg.rsf,
                         ids2, wts2)
    torch.cuda.synchronize()
    assert capi.device_error() == 0
    return logits.cpu().numpy(), ids.cpu().numpy(), wts.cpu().numpy(), ids2.cpu().numpy(), wts2.cpu().numpy()


def _check(cfg, x, w, lb, cb=None, rows=None):
    logits, ids, wts, ids2, wts2 = _gpu(x, w, lb, cb, cfg)
    x, w = x.cpu(), w.cpu()
    lb = None if lb is None else lb.cpu()
    rows = np.arange(x.shape[0]) if rows is None else np.asarray(rows)
    ref = oracle.router_logits(x.double().numpy()[rows], w.double().numpy(),
                               None if lb is None else lb.numpy())
    assert np.array_equal(logits[rows], ref), "logits differ from the fixed-order oracle sum"
    assert np.array_equal(ids, ids2) and np.array_equal(wts, wts2)
    check_routing(cfg, ref, None if cb is None else cb.numpy(), ids[rows], wts[rows])


SOFT = configs.small(configs.DECODE_BF16, name="rg_soft", T=32, H=2048, E=128, top_k=8)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_router_gemm_decode_shape(cuda_lib, dtype):
    x, w, lb = _inputs(32, 2048, 128, dtype, seed=11)
    _check(SOFT, x, w, lb)


@pytest.mark.parametrize("T,H,E,k", [(33, 256, 8, 2), (1, 512, 40, 3), (7, 1024, 64, 6), (5, 7168, 512, 8)])
def test_router_gemm_shapes(cuda_lib, T, H, E, k):
    cfg = configs.small(SOFT, name="rg_shape", T=T, H=H, E=E, top_k=k)
    x, w, lb = _inputs(T, H, E, "bf16", seed=T + H + E)
    _check(cfg, x, w, lb)


def test_router_gemm_without_bias_and_not_renormalised(cuda_lib):
    cfg = configs.small(SOFT, name="rg_norenorm", T=12, H=512, E=64, top_k=4, renormalize=False)
    x, w, _ = _inputs(12, 512, 64, "bf16", seed=3)
    _check(cfg, x, w, None)


def test_router_gemm_grouped_sigmoid(cuda_lib):
    cfg = configs.small(configs.FP8_A8W8, name="rg_grouped", T=64, H=4096, E=64, top_k=6)
    x, w, lb = _inputs(64, 4096, 64, "bf16", seed=5, bias_std=0.1)
    cb = torch.randn(64, generator=torch.Generator().manual_seed(6)) * 0.1
    _check(cfg, x, w, lb, cb)


def test_router_gemm_prefill_shape_sampled_rows(cuda_lib):
    # the MXFP8 prefill router: T = 4096, H = 7168, E = 256, grouped 8/4, Zipf
    # logit bias; every token routed on the GPU, 16 rows checked on the CPU
    cfg = configs.MXFP8_PREFILL
    inp = synth.make_layer_inputs(configs.small(cfg, name="rg_mx_small", I=128, Is=128), device="cuda")
    rows = np.sort(np.random.default_rng(2).choice(cfg.T, 16, replace=False))
    _check(cfg, inp["x_r"], inp["w_r"], inp["logit_bias"], rows=rows)


def test_layer_with_fused_router(cuda_lib):
    """The decode layer started from the router linear: the logits it used
    equal the oracle's, and the layer output matches the oracle fed with them."""
    cfg = configs.small(configs.DECODE_BF16, name="rg_layer", T=32, H=512, E=32, top_k=4, I=128, Is=128)
    inp = synth.make_layer_inputs(cfg)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    from routed_shared_experts_b200.layer import MoELayer
    layer = MoELayer(cfg, dev, router_gemm=True)
    layer.forward()
    torch.cuda.synchronize()
    assert capi.device_error() == 0
    ref_logits = oracle.router_logits(inp["x_r"].double().numpy(), inp["w_r"].double().numpy(),
                                      inp["logit_bias"].numpy())
    assert np.array_equal(layer.logits.cpu().numpy(), ref_logits)
    cpu = dict(synth.oracle_view(inp), logits=torch.from_numpy(ref_logits))
    agree = check_routing(cfg, ref_logits, None, layer.topk_ids.cpu().numpy(), layer.topk_weights.cpu().numpy())
    ref = oracle.moe_layer(cfg.as_dict(), cpu, tokens=agree)
    out = layer.out.float().cpu().numpy()[agree]
    assert_close_rms(out, ref["out"], BF16_TOL, "out", rounded=[ref["out"], ref["addend"]])
