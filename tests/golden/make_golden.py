"""Writes the oracle's results on three tiny seeded layers to tests/golden/.

    python tests/golden/make_golden.py

The pages print no worked example of the layer, so these fixtures are not the
pages' numbers: they freeze the oracle's own results (routing ids and weights,
the bf16 outputs) on small inputs from the seeded generator, so that any later
change to the oracle's arithmetic shows up as a fixture diff that has to be
justified. Only ``oracle/`` and the input generator are called.
"""
from __future__ import annotations

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from routed_shared_experts_b200 import configs, synth  # noqa: E402

CASES = {
    "tiny_layer_bf16": configs.small(configs.TINY_BF16, name="golden_bf16", T=6),
    "tiny_layer_fp8": configs.small(configs.FP8_A8W8, name="golden_fp8", T=6, H=256, E=8, top_k=2, I=128, Is=256,
                                    n_group=4, topk_group=2, block_m=16),
    "tiny_layer_mxfp4": configs.small(configs.MXFP4_PREFILL, name="golden_mxfp4", T=6, H=256, E=8, top_k=2, I=128,
                                      Is=128, n_group=4, topk_group=2, block_m=16),
}


def compute(cfg) -> dict:
    inp = synth.oracle_view(synth.make_layer_inputs(cfg))
    r = oracle.moe_layer(cfg.as_dict(), inp)
    return {
        "config": cfg.as_dict(),
        "topk_ids": r["topk_ids"].astype(int).tolist(),
        "topk_weights": [[float(v).hex() for v in row] for row in r["topk_weights"]],
        "out": [[float(v).hex() for v in row] for row in r["out"]],
    }


def main():
    for name, cfg in CASES.items():
        with open(os.path.join(HERE, name + ".json"), "w") as f:
            json.dump(compute(cfg), f)
            f.write("\n")
        print("wrote", name)


if __name__ == "__main__":
    main()
