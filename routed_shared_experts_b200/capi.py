"""ctypes binding of ``libmoe_b200.so`` (C ABI in ``include/moe_b200.h``).

Argument marshalling only: each function takes torch tensors (device memory)
and plain numbers, checks device and contiguity, and calls the C entry point of
the same name on the current (or given) CUDA stream. A non-zero status raises
``MoEError``. There is no fallback: if the library is not built, the first call
raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

MOE_OK = 0
MOE_DT_BF16, MOE_DT_FP16, MOE_DT_FP8_E4M3, MOE_DT_MXFP8_E4M3, MOE_DT_F32, MOE_DT_MXFP4_E2M1 = 0, 1, 2, 3, 4, 5
MOE_ROUTE_SOFTMAX, MOE_ROUTE_GROUPED_SIGMOID = 0, 1
# block-scaled layer formats (MXFP4 layers keep MXFP8 activations)
MX_FORMATS = ("mxfp8", "mxfp4")
DTYPES = {"bf16": MOE_DT_BF16, "fp16": MOE_DT_FP16, "fp8": MOE_DT_FP8_E4M3, "mxfp8": MOE_DT_MXFP8_E4M3,
          "mxfp4": MOE_DT_MXFP4_E2M1,
          "f32": MOE_DT_F32}
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

# name -> (restype, argtypes)
_P, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [_I]),
    "moe_version": (ctypes.c_char_p, []),
    "moe_last_cuda_error": (ctypes.c_char_p, []),
    "moe_supports_output_addend": (_I, []),
    "moe_device_error": (_I, [ctypes.POINTER(ctypes.c_int), _P]),
    "moe_selftest_wait_timeout": (_I, [_P]),
    "moe_sorted_capacity": (_SZ, [_I, _I, _I, _I]),
    "moe_stage2_workspace_bytes": (_SZ, [_I, _I]),
    "moe_stage1_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "moe_mx_weight_scale_bytes": (_SZ, [_I, _I, _I, _I]),
    "moe_mx_h_scale_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "moe_mx_pack_weight_scales": (_I, [_I, _P, _P, _I, _I, _I, _P]),
    "moe_router_topk": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P]),
    "moe_router_gemm_topk": (_I, [_I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _P]),
    "moe_align_sort": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "moe_stage1_gemm": (_I, [_I, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "moe_stage2_gemm_accumulate": (_I, [_I, _P, _P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P,
                                        _P, _P, _P]),
    "moe_stage2_gemm_accumulate_static_ws": (_I, [_I, _P, _P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                                  _P, _P, _P, _P]),
    "shared_expert_gate_dot": (_I, [_I, _P, _P, _I, _I, _I, _P, _P]),
    "moe_quantize_activations": (_I, [_I, _P, _I, _I, _P, _P, _P]),
    "moe_append_shared_slots": (_I, [_P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P]),
}

_LIB = None


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        lib_ = lib()
        msg = lib_.moe_status_string(status).decode()
        cuda = lib_.moe_last_cuda_error().decode()
        super().__init__(f"{fn}: {msg}" + (f" ({cuda})" if status in (-5, -7) and cuda else ""))
        self.status = status


def lib() -> ctypes.CDLL:
    """Load the library (once). Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m routed_shared_experts_b200.build")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor or None")
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _event(ev):
    if ev is None:
        return None
    return ev.cuda_event or None


def _check(name: str, status: int):
    if status != MOE_OK:
        raise MoEError(name, status)


def sorted_capacity(T: int, top_k: int, E: int, block_m: int) -> int:
    return lib().moe_sorted_capacity(T, top_k, E, block_m)


def stage2_workspace_bytes(T: int, H: int) -> int:
    return lib().moe_stage2_workspace_bytes(T, H)


def stage1_workspace_bytes(dtype: int, T: int, top_k: int, E: int, H: int, I: int, block_m: int) -> int:
    return lib().moe_stage1_workspace_bytes(dtype, T, top_k, E, H, I, block_m)


def mx_weight_scale_bytes(which: int, E: int, H: int, I: int) -> int:
    return lib().moe_mx_weight_scale_bytes(which, E, H, I)


def mx_h_scale_bytes(T: int, top_k: int, E: int, I: int, block_m: int) -> int:
    return lib().moe_mx_h_scale_bytes(T, top_k, E, I, block_m)


def moe_mx_pack_weight_scales(which, src, dst, E, H, I, stream=None):
    _check("moe_mx_pack_weight_scales", lib().moe_mx_pack_weight_scales(
        which, _ptr(src), _ptr(dst), E, H, I, _stream(stream)))


def device_error(stream=None) -> int:
    code = ctypes.c_int(0)
    _check("moe_device_error", lib().moe_device_error(ctypes.byref(code), _stream(stream)))
    return code.value


def moe_selftest_wait_timeout(stream=None):
    """Launch the bounded-wait self-test (device error 1 after ~4 s)."""
    _check("moe_selftest_wait_timeout", lib().moe_selftest_wait_timeout(_stream(stream)))


def moe_router_topk(logits, correction_bias, top_k, mode, n_group, topk_group, renormalize,
                    routed_scaling_factor, topk_ids, topk_weights, stream=None):
    T, E = logits.shape
    _check("moe_router_topk", lib().moe_router_topk(
        _ptr(logits), _ptr(correction_bias), T, E, top_k, mode, n_group, topk_group, int(renormalize),
        float(routed_scaling_factor), _ptr(topk_ids), _ptr(topk_weights), _stream(stream)))


def moe_router_gemm_topk(x, w_r, logit_bias, correction_bias, top_k, mode, n_group, topk_group, renormalize,
                         routed_scaling_factor, logits, topk_ids, topk_weights, stream=None):
    T, H = x.shape
    E = w_r.shape[1]
    dtype = MOE_DT_BF16 if x.dtype == torch.bfloat16 else MOE_DT_FP16
    _check("moe_router_gemm_topk", lib().moe_router_gemm_topk(
        dtype, _ptr(x), _ptr(w_r), _ptr(logit_bias), _ptr(correction_bias), T, H, E, top_k, mode, n_group,
        topk_group, int(renormalize), float(routed_scaling_factor), _ptr(logits), _ptr(topk_ids),
        _ptr(topk_weights), _stream(stream)))


def moe_align_sort(topk_ids, E, block_m, sorted_ids, block_expert, expert_counts, expert_offsets, num_padded,
                   stream=None):
    T, k = topk_ids.shape
    _check("moe_align_sort", lib().moe_align_sort(
        _ptr(topk_ids), T, k, E, block_m, _ptr(sorted_ids), _ptr(block_expert), _ptr(expert_counts),
        _ptr(expert_offsets), _ptr(num_padded), _stream(stream)))


def moe_stage1_gemm(dtype, x, x_scale, w13, w13_scale, sorted_ids, block_expert, num_padded, T, top_k, H, I, E,
                    block_m, h, h_scale, ws, stream=None):
    _check("moe_stage1_gemm", lib().moe_stage1_gemm(
        dtype, _ptr(x), _ptr(x_scale), _ptr(w13), _ptr(w13_scale), _ptr(sorted_ids), _ptr(block_expert),
        _ptr(num_padded), T, top_k, H, I, E, block_m, _ptr(h), _ptr(h_scale), _ptr(ws), _stream(stream)))


def moe_stage2_gemm_accumulate(dtype, h, h_scale, w2, w2_scale, weights, weights_dtype, sorted_ids, block_expert,
                               num_padded, T, top_k, H, I, E, block_m, addend, addend_ready, acc_ws, out,
                               stream=None):
    _check("moe_stage2_gemm_accumulate", lib().moe_stage2_gemm_accumulate(
        dtype, _ptr(h), _ptr(h_scale), _ptr(w2), _ptr(w2_scale), _ptr(weights), weights_dtype,
        _ptr(sorted_ids), _ptr(block_expert), _ptr(num_padded), T, top_k, H, I, E, block_m, _ptr(addend),
        _event(addend_ready), _ptr(acc_ws), _ptr(out), _stream(stream)))


def moe_stage2_gemm_accumulate_static_ws(dtype, h, h_scale, w2, w2_scale, weights, weights_dtype, sorted_ids,
                                         block_expert, num_padded, T, top_k, H, I, E, block_m, addend,
                                         addend_ready, out, stream=None):
    """Stage 2 with the library's own static workspace (no device allocation
    by the caller or the library); see include/moe_b200.h for its limit."""
    _check("moe_stage2_gemm_accumulate_static_ws", lib().moe_stage2_gemm_accumulate_static_ws(
        dtype, _ptr(h), _ptr(h_scale), _ptr(w2), _ptr(w2_scale), _ptr(weights), weights_dtype,
        _ptr(sorted_ids), _ptr(block_expert), _ptr(num_padded), T, top_k, H, I, E, block_m, _ptr(addend),
        _event(addend_ready), _ptr(out), _stream(stream)))


def moe_append_shared_slots(topk_ids, topk_weights, E, m, gate, out_ids, out_weights, stream=None):
    T, k = topk_ids.shape
    gdt = MOE_DT_FP16 if (gate is not None and gate.dtype == torch.float16) else MOE_DT_BF16
    _check("moe_append_shared_slots", lib().moe_append_shared_slots(
        _ptr(topk_ids), _ptr(topk_weights), T, k, E, m, _ptr(gate), gdt, _ptr(out_ids), _ptr(out_weights),
        _stream(stream)))


def moe_quantize_activations(dtype, x, codes, scale, stream=None):
    T, H = x.shape
    _check("moe_quantize_activations", lib().moe_quantize_activations(
        dtype, _ptr(x), T, H, _ptr(codes), _ptr(scale), _stream(stream)))


def shared_expert_gate_dot(dtype, x, w, apply_sigmoid, out, stream=None):
    T, K = x.shape
    _check("shared_expert_gate_dot", lib().shared_expert_gate_dot(
        dtype, _ptr(x), _ptr(w), T, K, int(apply_sigmoid), _ptr(out), _stream(stream)))
