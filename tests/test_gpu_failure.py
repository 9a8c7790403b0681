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
