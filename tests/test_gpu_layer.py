"""Parity of the full layer (five C-ABI calls, shared expert on a side stream)
and of the grouped-GEMM stages with the CPU oracle.

bf16 layers: max|out - ref| <= 1e-2 * rms(ref); routing ids, the sort and the
gate compared as in the kernel tests."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import BF16_TOL, assert_close_rms, oracle_layer, run_layer, to_dev
from routed_shared_experts_b200 import capi, configs, synth
from routed_shared_experts_b200.layer import MoELayer

pytestmark = pytest.mark.gpu

# Reduced decode layer spanning several weight tiles in both stages (H = 3 x 128,
# I = 3 x 64) and several token blocks per hot expert, with a ragged last block.
MULTI = configs.small(configs.DECODE_BF16, name="multi_bf16", T=53, H=384, E=16, top_k=4, I=192, Is=128,
                      seed=11)


def _check_layer(cfg, block_m=None, tokens=None):
    inp = synth.make_layer_inputs(cfg)
    layer = run_layer(cfg, to_dev(inp), block_m=block_m)
    ref = oracle_layer(cfg, inp, tokens=tokens)
    tok = ref["tokens"]
    assert np.array_equal(layer.topk_ids.cpu().numpy(), ref["topk_ids"])
    np.testing.assert_allclose(layer.topk_weights.cpu().numpy(), ref["topk_weights"], rtol=1e-6)
    srt = oracle.align_sort(ref["topk_ids"], cfg.E, block_m or cfg.block_m)
    n = int(layer.num_padded.item())
    assert n == srt["num_padded"]
    assert np.array_equal(layer.sorted_ids.cpu().numpy()[:n], srt["sorted_ids"])
    if cfg.shared_gate:
        g = layer.gate.float().cpu().numpy()[tok]
        assert np.all(np.abs(g - ref["gate"]) <= 2.0**-8 * np.abs(ref["gate"]) + 1e-12)
    add = layer.addend.float().cpu().numpy()[tok]
    assert_close_rms(add, ref["addend"], BF16_TOL, "addend", exact_frac=0.9)
    out = layer.out.float().cpu().numpy()[tok]
    rel = assert_close_rms(out, ref["out"], BF16_TOL, "out", rounded=[ref["out"], ref["addend"]],
                           exact_frac=0.9)
    # the stage-2 workspace is left zeroed for the next call
    assert torch.count_nonzero(layer.acc_ws).item() == 0
    return layer, ref, rel


def test_layer_tiny_bf16(cuda_lib):
    _check_layer(configs.TINY_BF16)


def test_layer_decode_bf16(cuda_lib):
    _check_layer(configs.DECODE_BF16)


@pytest.mark.parametrize("block_m", [16, 32, 64, 128, 256])
def test_layer_block_sizes(cuda_lib, block_m):
    _check_layer(MULTI, block_m=block_m)


@pytest.mark.parametrize("kw", [dict(T=1), dict(T=1, top_k=1), dict(E=1, top_k=1), dict(top_k=16),
                                dict(T=200, E=4, top_k=2), dict(T=17, H=128, I=64, Is=64)])
def test_layer_edge_shapes(cuda_lib, kw):
    _check_layer(configs.small(MULTI, **kw))


def test_stage1_hidden_matches_oracle(cuda_lib):
    cfg = MULTI
    inp = synth.make_layer_inputs(cfg)
    layer = run_layer(cfg, to_dev(inp))
    h = layer.h.float().cpu().numpy()
    s = layer.sorted_ids.cpu().numpy()
    be = layer.block_expert.cpu().numpy()
    n = int(layer.num_padded.item())
    x = inp["x"].double().numpy()
    for r in range(n):
        f = s[r]
        if f >= cfg.T * cfg.top_k:
            continue
        e = be[r // cfg.block_m]
        ref = oracle.bf16_round(oracle.expert_hidden(x[f // cfg.top_k], inp["w13"][e].double().numpy(), cfg.I))
        np.testing.assert_allclose(h[r], ref, rtol=2.0**-7, atol=1e-5 * np.abs(ref).max())
    # shared expert stage 1 (identity routing)
    hs = layer.h_s.float().cpu().numpy()
    for t in range(cfg.T):
        ref = oracle.bf16_round(oracle.expert_hidden(x[t], inp["w13s"].double().numpy(), cfg.Is))
        np.testing.assert_allclose(hs[t], ref, rtol=2.0**-7, atol=1e-5 * np.abs(ref).max())


def test_addend_in_epilogue_equals_separate_add(cuda_lib):
    """Accumulating the shared output in the stage-2 epilogue equals routing
    without the addend followed by a separate add (within the bf16 bound)."""
    cfg = MULTI
    inp = to_dev(synth.make_layer_inputs(cfg))
    layer = MoELayer(cfg, inp)
    layer.forward()
    fused = layer.out.float().clone()
    main = torch.cuda.current_stream()
    layer.routed(main, addend=False)
    torch.cuda.synchronize()
    routed = layer.out.float().cpu().numpy()
    addend = layer.addend.float().cpu().numpy()
    # fused rounds (addend + routed sum) once; the separate path rounded the
    # routed sum first: one bf16 step of each may separate them
    assert_close_rms(fused.cpu().numpy(), routed + addend, BF16_TOL, "fused vs separate",
                     rounded=[routed + addend, routed], mean_check=False)


def test_rsf_fold_scales_routed_output(cuda_lib):
    """routed_scaling_factor folded into the weights scales the routed part."""
    base = configs.small(MULTI, shared_gate=False)
    inp = to_dev(synth.make_layer_inputs(base))
    outs = []
    for rsf in (1.0, 2.5):
        layer = MoELayer(configs.small(base, rsf=rsf), inp)
        layer.routed(torch.cuda.current_stream(), addend=False)
        torch.cuda.synchronize()
        outs.append(layer.out.float().cpu().numpy())
    assert_close_rms(outs[1], 2.5 * outs[0], BF16_TOL, "rsf fold", rounded=[outs[1], 2.5 * outs[0]],
                     mean_check=False)


def test_cuda_graph_replay(cuda_lib):
    cfg = MULTI
    inp = to_dev(synth.make_layer_inputs(cfg))
    layer = MoELayer(cfg, inp)
    layer.forward()
    torch.cuda.synchronize()
    eager = layer.out.float().clone()
    s = torch.cuda.Stream()
    graph = layer.capture(s)
    with torch.cuda.stream(s):
        for _ in range(3):
            graph.replay()
    torch.cuda.synchronize()
    assert capi.device_error() == 0
    assert_close_rms(layer.out.float().cpu().numpy(), eager.cpu().numpy(), BF16_TOL, "graph vs eager",
                     exact_frac=0.95)
    assert torch.count_nonzero(layer.acc_ws).item() == 0
    del graph


def test_repeated_steps_are_stable(cuda_lib):
    cfg = configs.DECODE_BF16
    inp = synth.make_layer_inputs(cfg)
    layer = run_layer(cfg, to_dev(inp), steps=5)
    ref = oracle_layer(cfg, inp, tokens=np.arange(0, cfg.T, 4))
    assert_close_rms(layer.out.float().cpu().numpy()[ref["tokens"]], ref["out"], BF16_TOL, "after 5 steps",
                     rounded=[ref["out"], ref["addend"]], exact_frac=0.9)
