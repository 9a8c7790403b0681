"""CPU oracle of the routed + shared-expert MoE layer (test infrastructure).

Only the test suite, the smoke check and the benchmark's CPU-baseline legs use
this package; the GPU library never imports it.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import (  # noqa: F401
    BF16, E2M1_TABLE, E4M3, E4M3_MAX, FP16, FP32, align_sort, bf16_round, decode_operand, e2m1_decode, e2m1_unpack,
    e4m3_decode, e4m3_encode,
    expert_forward, expert_hidden, moe_layer, mx_block_exponent, quantize_activations, quantize_h, round_to_format,
    route,
    router_grouped_sigmoid_topk, router_logits, router_softmax_topk, shared_pieces, shared_gate, sigmoid_fp32,
    sigmoid_fp32_hazard_mask, sigmoid_fp32_hazards, sigmoid_fp32_other, silu, sorted_capacity, tolerance_ok, ue8m0_decode,
)
