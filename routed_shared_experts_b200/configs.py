"""Workload table of the routed + shared-expert MoE layer.

Each entry is a synthetic layer: sizes, number format, routing mode and seed.
Names say what the workload is:

* ``tiny_bf16``      T=16   H=256  E=8   k=2 I=128  Is=128  softmax, gated shared expert
* ``decode_bf16``    T=32   H=2048 E=128 k=8 I=768  Is=512  softmax + N(0,0.5) logit bias, gated
* ``fp8_a8w8``       T=1024 H=4096 E=64  k=6 I=1408 Is=2816 grouped sigmoid 8/4, rsf 2.5
* ``mxfp8_prefill``  T=4096 H=7168 E=256 k=8 I=2048 Is=2048 grouped sigmoid 8/4, Zipf logit bias
* ``fp8_decode_T{n}`` the fp8_a8w8 shapes at T in {1,2,4,...,128}
* ``mxfp4_decode``   the decode_bf16 shapes (no shared gate) with MXFP4 weights, MXFP8 activations
* ``mxfp4_prefill``  the mxfp8_prefill shapes with MXFP4 weights, MXFP8 activations
"""
from __future__ import annotations

from dataclasses import asdict, dataclass, replace


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    H: int
    E: int
    top_k: int
    I: int
    Is: int
    dtype: str            # 'bf16' | 'fp8' (per-token x scale, per-expert W scale) | 'mxfp8'
                          # | 'mxfp4' (e2m1 weights, MXFP8 activations)
    route: str            # 'softmax' | 'grouped_sigmoid'
    seed: int
    block_m: int          # sort padding / token tile of the grouped GEMMs
    n_group: int = 1
    topk_group: int = 1
    rsf: float = 1.0      # routed_scaling_factor, folded into the top-k weights
    renormalize: bool = True
    shared_gate: bool = False
    logit_bias: str = "none"          # 'none' | 'normal0.5' | 'zipf1.2'
    correction_bias_std: float = 0.0  # grouped-sigmoid choice bias ~ N(0, std)
    weight_std: float = 0.02

    def as_dict(self) -> dict:
        return asdict(self)

    @property
    def has_correction_bias(self) -> bool:
        return self.correction_bias_std > 0


TINY_BF16 = MoEConfig("tiny_bf16", T=16, H=256, E=8, top_k=2, I=128, Is=128, dtype="bf16",
                      route="softmax", seed=0, block_m=16, shared_gate=True)
DECODE_BF16 = MoEConfig("decode_bf16", T=32, H=2048, E=128, top_k=8, I=768, Is=512, dtype="bf16",
                        route="softmax", seed=1, block_m=16, shared_gate=True,
                        logit_bias="normal0.5")
FP8_A8W8 = MoEConfig("fp8_a8w8", T=1024, H=4096, E=64, top_k=6, I=1408, Is=2816, dtype="fp8",
                     route="grouped_sigmoid", seed=2, block_m=128, n_group=8, topk_group=4,
                     rsf=2.5, correction_bias_std=0.1)
MXFP8_PREFILL = MoEConfig("mxfp8_prefill", T=4096, H=7168, E=256, top_k=8, I=2048, Is=2048,
                          dtype="mxfp8", route="grouped_sigmoid", seed=3, block_m=128,
                          n_group=8, topk_group=4, logit_bias="zipf1.2")

MXFP4_DECODE = MoEConfig("mxfp4_decode", T=32, H=2048, E=128, top_k=8, I=768, Is=512, dtype="mxfp4",
                         route="softmax", seed=6, block_m=16, logit_bias="normal0.5")
MXFP4_PREFILL = replace(MXFP8_PREFILL, name="mxfp4_prefill", dtype="mxfp4", seed=5)

SWEEP_T = (1, 2, 4, 8, 16, 32, 64, 128)


def fp8_decode(T: int) -> MoEConfig:
    """The fp8 a8w8 layer shapes at a decode batch of T tokens."""
    return replace(FP8_A8W8, name=f"fp8_decode_T{T}", T=T, seed=4, block_m=16)


GATE_K = (1024, 2048, 4096)
GATE_DTYPES = ("bf16", "fp16")
GATE_SEED = 4

CONFIGS = {c.name: c for c in (TINY_BF16, DECODE_BF16, FP8_A8W8, MXFP8_PREFILL, MXFP4_DECODE, MXFP4_PREFILL)}
CONFIGS.update({fp8_decode(t).name: fp8_decode(t) for t in SWEEP_T})


def small(cfg: MoEConfig, **kw) -> MoEConfig:
    """A reduced copy of a config (used for parity cases the oracle finishes in
    seconds while still spanning several tiles and a ragged tail)."""
    return replace(cfg, **kw)
