"""StepPipeline (overlapped host copies, graph-replayed steps) against one
eager step per batch: the same layer fed five different host batches must give
the same outputs either way (the fp32 reduction order of stage 2 may move a
few outputs by one bf16 step)."""
import pytest
import torch

from gpu_helpers import BF16_TOL, FP8_TOL, assert_close_rms, to_dev
from routed_shared_experts_b200 import capi, configs, synth
from routed_shared_experts_b200.layer import FusedSharedMoELayer, MoELayer
from routed_shared_experts_b200.pipeline import StepPipeline

pytestmark = pytest.mark.gpu


def _batches(cfg, names, n, seed):
    """n host batches of the named inputs: the layer's own inputs with their
    token rows permuted (a different batch per step, same formats)."""
    g = torch.Generator().manual_seed(seed)
    base = synth.make_layer_inputs(cfg)
    out = []
    for _ in range(n):
        perm = torch.randperm(cfg.T, generator=g)
        out.append([base[k][perm].contiguous().pin_memory() for k in names])
    return out


@pytest.mark.parametrize("name,fused", [("tiny_bf16", False), ("fp8_decode_T8", False), ("tiny_bf16", True)])
def test_pipeline_equals_eager_steps(cuda_lib, name, fused):
    cfg = configs.CONFIGS[name]
    inp = to_dev(synth.make_layer_inputs(cfg))
    layer = (FusedSharedMoELayer if fused else MoELayer)(cfg, inp)
    names = ["x"] + (["x_scale"] if inp.get("x_scale") is not None else []) + ["logits"]
    batches = _batches(cfg, names, 5, seed=7)
    ref = []
    for hb in batches:
        for k, t in zip(names, hb):
            inp[k].copy_(t)
        layer.forward()
        torch.cuda.synchronize()
        ref.append(layer.out.float().cpu().clone())
    pipe = StepPipeline(layer, names)
    outs = [torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory() for _ in batches]
    done = pipe.run(batches, outs)
    done.synchronize()
    assert capi.device_error() == 0
    tol = BF16_TOL if cfg.dtype == "bf16" else FP8_TOL
    for i, (o, r) in enumerate(zip(outs, ref)):
        assert_close_rms(o.float().numpy(), r.numpy(), tol, f"step {i}", exact_frac=0.95)
