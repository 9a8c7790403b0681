"""CPU oracle of the routed + shared-expert MoE layer (test infrastructure).

Only the test suite, the smoke check and the benchmark's CPU legs use this
package; the GPU library never imports it.

The oracle of record is the plain C++17 implementation (``moe_oracle.cpp``,
built into ``liboracle.so`` and bound by ``oracle.cpp``); the names below come
from it. ``oracle.np_oracle`` is an independent float64 numpy statement of the
same definitions, kept as a second opinion: the pins run against both.
"""
from . import moe_oracle as np_oracle  # noqa: F401
from .cpp import (  # noqa: F401
    BF16, E4M3, E4M3_MAX, FP16, FP32, align_sort, bf16_round, build, decode_operand, e2m1_decode, e2m1_unpack,
    e4m3_decode, e4m3_encode, expert_forward, expert_hidden, fp16_round, fp32_round, moe_layer, mx_block_exponent,
    num_threads, quantize_activations, quantize_h, round_to_format, route, router_grouped_sigmoid_topk,
    router_logits, router_softmax_topk, shared_gate, shared_pieces, sigmoid_fp32, sigmoid_fp32_hazard_mask,
    sigmoid_fp32_hazards, sigmoid_fp32_other, silu, sorted_capacity, tolerance_ok, ue8m0_decode,
)
