"""Failure detection without a GPU fault: a bounded wait that runs out
records its status in the device error word, the kernel returns, and the
context stays usable for the next layer step."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import BF16_TOL, assert_close_rms, to_dev
from routed_shared_experts_b200 import capi, configs, synth
from routed_shared_experts_b200.layer import MoELayer

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives(cuda_lib):
    assert capi.device_error() == 0
    capi.moe_selftest_wait_timeout()
    assert capi.device_error() == 1        # kErrWaitTimeout, read and cleared
    assert capi.device_error() == 0
    cfg = configs.TINY_BF16
    inp = synth.make_layer_inputs(cfg)
    layer = MoELayer(cfg, to_dev(inp))
    layer.forward()
    torch.cuda.synchronize()
    assert capi.device_error() == 0
    ref = oracle.moe_layer(cfg.as_dict(), synth.oracle_view(inp))
    assert np.array_equal(layer.topk_ids.cpu().numpy(), ref["topk_ids"])
    assert_close_rms(layer.out.float().cpu().numpy(), ref["out"], BF16_TOL, "out after the timeout")


@pytest.mark.parametrize("block_m", [16, 128])
def test_block_expert_out_of_range_is_reported_not_followed(cuda_lib, block_m):
    """A block_expert entry outside [0, E) (a stale or foreign buffer) makes
    the GEMMs record device error 4 and compute that block with expert 0's
    weights, so no load leaves the weight tensors; the other blocks are
    unaffected. The bad entry is planted on the host into a sort result that
    is otherwise valid; the kernels' own range check turns it into the error."""
    cfg = configs.small(configs.DECODE_BF16, name="bad_expert", T=40, H=512, E=8, top_k=2, I=256, Is=128, seed=17,
                        block_m=block_m)
    inp = to_dev(synth.make_layer_inputs(cfg))
    layer = MoELayer(cfg, inp)
    layer.forward()
    torch.cuda.synchronize()
    assert capi.device_error() == 0
    good_h = layer.h.clone()
    n_blocks = int(layer.num_padded.item()) // block_m
    be = layer.block_expert.clone()
    bad = n_blocks - 1
    be[bad] = cfg.E + 3
    h = torch.zeros_like(layer.h)
    capi.moe_stage1_gemm(layer.dt, inp["x"], None, inp["w13"], None, layer.sorted_ids, be, layer.num_padded,
                         cfg.T, cfg.top_k, cfg.H, cfg.I, cfg.E, block_m, h, None, layer.ws1)
    torch.cuda.synchronize()
    assert capi.device_error() == 4
    assert capi.device_error() == 0
    # rows of the blocks before the planted one that hold a slot (the rest of a
    # short block is never written): as computed from the true sort
    srt = layer.sorted_ids[: bad * block_m]
    rows = torch.nonzero(srt < cfg.T * cfg.top_k).flatten()
    assert torch.equal(h[rows], good_h[rows])
    # the context stays usable: a full step afterwards is clean
    layer.forward()
    torch.cuda.synchronize()
    assert capi.device_error() == 0
