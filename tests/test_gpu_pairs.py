"""The grouped GEMMs on CTA pairs (2-CTA clusters, one M = 256 tcgen05 MMA
per pair; selected with MOE_B200_PAIR=1, read once per process) against the
C++ oracle: bf16, fp8 (stage 2 on pairs, stage 1 on single CTAs) and MXFP8 /
MXFP4 layers with 128- and 16-token blocks (H = 640: a last stage of one K
atom), full and short token tiles, and the bf16 decode layer, run in a child
process so that the choice is made fresh."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + '/tests')
import oracle
from gpu_helpers import (BF16_TOL, FP8_TOL, assert_close_rms, check_routing, quantised_layer_allowance, run_layer,
                         to_dev)
from routed_shared_experts_b200 import configs, synth
res = {}
cases = {
    "bf16": configs.small(configs.DECODE_BF16, name="pair_bf16", T=300, H=512, E=8, top_k=2, I=256, Is=256,
                          block_m=128, seed=51),
    "fp8": configs.small(configs.FP8_A8W8, name="pair_fp8", T=300, H=512, E=8, top_k=2, I=256, Is=256,
                         n_group=4, topk_group=2, block_m=128, seed=52),
    "mxfp8": configs.small(configs.MXFP8_PREFILL, name="pair_mx", T=300, H=512, E=8, top_k=2, I=256, Is=256,
                           n_group=4, topk_group=2, block_m=128, seed=53),
    "mxfp4": configs.small(configs.MXFP4_PREFILL, name="pair_mx4", T=300, H=512, E=8, top_k=2, I=256, Is=256,
                           n_group=4, topk_group=2, block_m=128, seed=54),
    # 16-token tiles (8 token rows per CTA of a pair, one M = 256, N = 16 MMA)
    "bf16_16": configs.small(configs.DECODE_BF16, name="pair_bf16_16", T=40, H=512, E=16, top_k=4, I=256, Is=256,
                             seed=55),
    "fp8_16": configs.small(configs.FP8_A8W8, name="pair_fp8_16", T=40, H=512, E=16, top_k=4, I=256, Is=256,
                            n_group=4, topk_group=2, block_m=16, seed=56),
    "mxfp8_16": configs.small(configs.MXFP8_PREFILL, name="pair_mx_16", T=40, H=640, E=16, top_k=4, I=256,
                              Is=256, n_group=4, topk_group=2, block_m=16, seed=57),
    "mxfp4_16": configs.small(configs.MXFP4_DECODE, name="pair_mx4_16", T=40, H=512, E=16, top_k=4, I=256, Is=256,
                              seed=58),
    "decode_bf16": configs.DECODE_BF16,
}
for name, cfg in cases.items():
    inp = synth.make_layer_inputs(cfg)
    layer = run_layer(cfg, to_dev(inp))
    cpu = synth.oracle_view(inp)
    bias = None if cpu.get("correction_bias") is None else cpu["correction_bias"].numpy()
    agree = check_routing(cfg, cpu["logits"].numpy(), bias, layer.topk_ids.cpu().numpy(),
                          layer.topk_weights.cpu().numpy())
    q = cfg.dtype != "bf16"
    ref = oracle.moe_layer(cfg.as_dict(), cpu, tokens=agree, want_h=q)
    tol = FP8_TOL if q else BF16_TOL
    allow_out = allow_add = None
    if q:
        allow_out, allow_add, _ = quantised_layer_allowance(cfg, layer, cpu, agree, ref)
    assert_close_rms(layer.addend.float().cpu().numpy()[agree], ref["addend"], tol, "addend", allow=allow_add)
    r = assert_close_rms(layer.out.float().cpu().numpy()[agree], ref["out"], tol, "out",
                         rounded=[ref["out"], ref["addend"]], allow=allow_out, exact_frac=0.9)
    res[name] = r
print("RESULT " + json.dumps(res))
"""


def test_pair_gemms_match_the_oracle(cuda_lib):
    env = dict(os.environ, MOE_B200_PAIR="1")
    code = CHILD.replace("ROOT", repr(ROOT), 2)
    p = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert p.returncode == 0, p.stdout[-3000:] + p.stderr[-3000:]
    line = [ln for ln in p.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    assert set(json.loads(line[7:])) == {"bf16", "fp8", "mxfp8", "mxfp4", "bf16_16", "fp8_16", "mxfp8_16",
                                         "mxfp4_16", "decode_bf16"}
