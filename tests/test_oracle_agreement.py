"""The two statements of the oracle - the plain C++ one of record and the
independent float64 numpy one - against each other on whole layers (CPU):
bf16, fp8 per-token/per-expert, MXFP8 and MXFP4 layers, softmax and biased
grouped sigmoid routing, both shared-expert modes. Routing ids, the shared
gate and the rounded outputs must agree bit for bit; top-k weights and the
unrounded routed sums to float64 round-off (the two use different exp and
summation orders)."""
import numpy as np
import pytest

import oracle
from oracle import moe_oracle as np_oracle
from routed_shared_experts_b200 import configs, synth

CASES = {
    "tiny_bf16": configs.TINY_BF16,
    "fp8": configs.small(configs.FP8_A8W8, name="agree_fp8", T=40, H=512, E=16, top_k=4, I=256, Is=384, n_group=4,
                         topk_group=2, block_m=32, seed=21),
    "mxfp8": configs.small(configs.MXFP8_PREFILL, name="agree_mx", T=30, H=512, E=8, top_k=2, I=256, Is=256,
                           n_group=4, topk_group=2, block_m=32, seed=31),
    "mxfp4": configs.small(configs.MXFP4_DECODE, name="agree_mx4", T=20, H=256, E=8, top_k=2, I=128, Is=128, seed=7),
    "decode_bf16": configs.small(configs.DECODE_BF16, name="agree_dec", T=8, H=512, E=32, top_k=4, I=256, Is=128,
                                 seed=11),
}


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("name", list(CASES))
def test_cpp_and_numpy_oracles_agree(name, fused):
    cfg = CASES[name]
    inp = synth.oracle_view(synth.make_layer_inputs(cfg))
    a = np_oracle.moe_layer(cfg.as_dict(), inp, shared_fused=fused)
    b = oracle.moe_layer(cfg.as_dict(), inp, shared_fused=fused)
    assert np.array_equal(a["topk_ids"], b["topk_ids"])
    assert np.array_equal(a["gate"], b["gate"])
    np.testing.assert_allclose(b["topk_weights"], a["topk_weights"], rtol=1e-14, atol=0)
    rms = np.sqrt(np.mean(a["routed"] ** 2))
    assert np.max(np.abs(a["routed"] - b["routed"])) <= 1e-14 * rms
    np.testing.assert_allclose(b["addend"], a["addend"], rtol=1e-14, atol=1e-16)
    assert np.array_equal(a["out"], b["out"])
