"""Python binding of the plain C++ oracle (``oracle/moe_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU legs of ``bench.py``; the product path never imports it.

The functions have the names and signatures of the float64 numpy oracle
(``oracle/moe_oracle.py``, kept as an independent second statement of the same
definitions); every computation happens in ``liboracle.so``. This module only
moves arrays in and out (argument marshalling). The library is built with
``build()`` (g++, C++17, OpenMP, no fast-math, no FP contraction) into
``oracle/liboracle.so``; it shares no source with the CUDA library.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.cpp")
LIB_PATH = os.path.join(HERE, "liboracle.so")

E4M3_MAX = 448.0
ROUTER_CHUNKS = 8
FMT_CODES = {"bf16": 0, "fp16": 1, "fp32": 2, "e4m3": 3}
LAYER_FMT = {"bf16": 0, "fp8": 1, "mxfp8": 2, "mxfp4": 3}


def build(force: bool = False) -> str:
    """Compile liboracle.so (portable x86-64 code: no -march=native, so the
    library also runs on a host with another CPU)."""
    if not force and os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= os.path.getmtime(SRC):
        return LIB_PATH
    cmd = ["g++", "-O3", "-std=c++17", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-o", LIB_PATH, SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("building the C++ oracle failed:\n" + res.stdout + res.stderr)
    return LIB_PATH


_LIB = None


class OrcLayer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("T", "H", "E", "top_k", "I", "Is", "fmt", "route", "n_group",
                                             "topk_group", "renormalize")] + [
        ("rsf", ctypes.c_double), ("shared_gate", ctypes.c_int),
        ("logits", ctypes.c_void_p), ("corr_bias", ctypes.c_void_p), ("x", ctypes.c_void_p),
        ("x_scale", ctypes.c_void_p), ("w_gate", ctypes.c_void_p), ("w13", ctypes.c_void_p),
        ("w13_scale", ctypes.c_void_p), ("w2", ctypes.c_void_p), ("w2_scale", ctypes.c_void_p),
        ("w13s", ctypes.c_void_p), ("w13s_scale", ctypes.c_void_p), ("w2s", ctypes.c_void_p),
        ("w2s_scale", ctypes.c_void_p)]


def lib():
    global _LIB
    if _LIB is None:
        build()
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        sigs = {
            "orc_round": (None, [P, P, i64, i32]),
            "orc_e4m3_decode": (None, [P, P, i64]),
            "orc_e2m1_decode": (None, [P, P, i64]),
            "orc_ue8m0_decode": (None, [P, P, i64]),
            "orc_bf16_decode": (None, [P, P, i64]),
            "orc_fp16_decode": (None, [P, P, i64]),
            "orc_mx_exponent": (None, [P, P, i64]),
            "orc_e4m3_encode": (i64, [P, P, i64]),
            "orc_decode_matrix": (None, [i32, P, P, i64, i32, P]),
            "orc_quantize_activations": (None, [P, i32, i32, i32, P, P]),
            "orc_quantize_h": (None, [P, i64, i32, i32]),
            "orc_silu": (None, [P, P, i64]),
            "orc_router_logits": (i32, [P, P, P, i32, i32, i32, i32, P]),
            "orc_router_softmax_topk": (None, [P, i32, i32, i32, i32, f64, P, P]),
            "orc_sigmoid_fp32": (None, [P, P, i64]),
            "orc_sigmoid_hazards": (None, [P, i64, i32, P, P]),
            "orc_router_grouped_topk": (None, [P, P, P, i32, i32, i32, i32, i32, i32, f64, P, P]),
            "orc_sorted_capacity": (i64, [i32, i32, i32, i32]),
            "orc_align_sort": (i32, [P, i32, i32, i32, i32, P, P, P, P, P]),
            "orc_shared_gate": (None, [P, P, i32, i32, i32, i32, P]),
            "orc_expert_forward": (None, [P, P, P, i32, i32, i32, f64, f64, f64, P, P]),
            "orc_moe_layer": (i32, [ctypes.POINTER(OrcLayer), P, i32, i32, i32, P, P, P, P, P, P]),
            "orc_moe_layer_h": (i32, [ctypes.POINTER(OrcLayer), P, i32, i32, i32, P, P, P, P, P, P, P, P, P, P]),
            "orc_layer_units": (i32, [ctypes.POINTER(OrcLayer), P, P, P, i32, i32, P]),
            "orc_num_threads": (i32, []),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


# ------------------------------------------------------------------ marshalling


def _np(t):
    """numpy view of a numpy array or CPU/GPU torch tensor (bf16 / fp16 as
    their 16-bit patterns, everything else as is)."""
    if isinstance(t, np.ndarray):
        return t
    try:
        import torch
    except ImportError:  # pragma: no cover
        return np.asarray(t)
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        if t.dtype == torch.float16:
            return t.view(torch.int16).numpy().view(np.uint16)
        if t.dtype == torch.float8_e4m3fn:
            return t.view(torch.uint8).numpy()
        return t.numpy()
    return np.asarray(t)


def _is_half(t, which):
    try:
        import torch
        return isinstance(t, torch.Tensor) and t.dtype == which
    except ImportError:  # pragma: no cover
        return False


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, np.float64))


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _values(t, fmt_hint=None):
    """float64 values of bf16 / fp16 tensors (decoded by the library from their
    bit patterns) or of plain numeric arrays."""
    try:
        import torch
        if isinstance(t, torch.Tensor) and t.dtype in (torch.bfloat16, torch.float16):
            bits = np.ascontiguousarray(_np(t))
            out = np.empty(bits.shape, np.float64)
            fn = lib().orc_bf16_decode if t.dtype == torch.bfloat16 else lib().orc_fp16_decode
            fn(_ptr(bits), _ptr(out), bits.size)
            return out
    except ImportError:  # pragma: no cover
        pass
    a = _np(t)
    if a.dtype == np.uint16 and fmt_hint in ("bf16", "fp16"):
        out = np.empty(a.shape, np.float64)
        bits = np.ascontiguousarray(a)
        (lib().orc_bf16_decode if fmt_hint == "bf16" else lib().orc_fp16_decode)(_ptr(bits), _ptr(out), bits.size)
        return out
    return _f64(a)


# ------------------------------------------------------------------ formats


class FloatFormat:
    def __init__(self, name):
        self.name = name


BF16, FP16, FP32, E4M3 = FloatFormat("bf16"), FloatFormat("fp16"), FloatFormat("fp32"), FloatFormat("e4m3")


def round_to_format(x, fmt) -> np.ndarray:
    """Nearest value of ``fmt`` (ties to even; e4m3 saturating)."""
    a = _f64(x)
    out = np.empty_like(a)
    lib().orc_round(_ptr(a), _ptr(out), a.size, FMT_CODES[fmt.name])
    return out.reshape(np.shape(x))


def bf16_round(x):
    return round_to_format(x, BF16)


def fp16_round(x):
    return round_to_format(x, FP16)


def fp32_round(x):
    return round_to_format(x, FP32)


def _decode(fn, codes, dtype=np.uint8):
    c = np.ascontiguousarray(np.asarray(codes, dtype))
    out = np.empty(c.shape, np.float64)
    fn(_ptr(c), _ptr(out), c.size)
    return out


def e4m3_decode(codes):
    return _decode(lib().orc_e4m3_decode, codes)


def e2m1_decode(codes):
    return _decode(lib().orc_e2m1_decode, codes)


def ue8m0_decode(b):
    return _decode(lib().orc_ue8m0_decode, b)


def mx_block_exponent(amax):
    a = _f64(amax)
    out = np.empty(a.shape, np.int32)
    lib().orc_mx_exponent(_ptr(a), _ptr(out), a.size)
    return out.astype(np.int64)


def e4m3_encode(values):
    v = _f64(values)
    out = np.empty(v.shape, np.uint8)
    bad = lib().orc_e4m3_encode(_ptr(v), _ptr(out), v.size)
    assert bad < 0, "not an e4m3 value"
    return out


def e2m1_unpack(packed):
    """Codes [..., 2n] of e2m1 values stored two per byte: element 2j in bits
    0-3, element 2j+1 in bits 4-7 (data layout only; no arithmetic)."""
    b = np.asarray(packed, np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def decode_operand(t, fmt: str, scale=None):
    """float64 values of a stored operand ('bf16' / 'fp16' tensors or bit
    patterns, 'fp8' e4m3 codes, 'mxfp8' codes + ue8m0 per 32 columns, 'mxfp4'
    e2m1 two per byte + ue8m0 per 32 unpacked columns)."""
    if fmt in ("bf16", "fp16"):
        return _values(t, fmt)
    a = np.ascontiguousarray(_np(t))
    code = {"fp8": 1, "mxfp8": 2, "mxfp4": 3}[fmt]
    cols = a.shape[-1] * (2 if fmt == "mxfp4" else 1)
    rows = int(np.prod(a.shape[:-1])) if a.ndim > 1 else 1
    sc = np.ascontiguousarray(_np(scale)) if scale is not None else None
    out = np.empty((rows, cols), np.float64)
    lib().orc_decode_matrix(code, _ptr(a), _ptr(sc), rows, cols, _ptr(out))
    return out.reshape(a.shape[:-1] + (cols,))


def quantize_activations(x, mode: str):
    """Codes uint8 [T, H] and scales (fp32 [T] for 'fp8', ue8m0 [T, H/32] for
    'mxfp8') of bf16 activations x [T, H]."""
    xv = _values(x)
    T, H = xv.shape
    codes = np.empty((T, H), np.uint8)
    if mode == "fp8":
        sc = np.empty(T, np.float32)
        m = 0
    elif mode == "mxfp8":
        assert H % 32 == 0
        sc = np.empty((T, H // 32), np.uint8)
        m = 1
    else:
        raise ValueError(mode)
    lib().orc_quantize_activations(_ptr(xv), T, H, m, _ptr(codes), _ptr(sc))
    return codes, sc


def quantize_h(h, mode: str) -> np.ndarray:
    a = _f64(h).copy()
    shape = a.shape
    n = shape[-1]
    lib().orc_quantize_h(_ptr(a), a.size // n, n, {"bf16": 0, "fp8": 1, "mxfp8": 2}[mode])
    return a.reshape(shape)


def silu(z):
    return _decode(lib().orc_silu, z, np.float64)


# ------------------------------------------------------------------ router


def router_logits(x, w_r, logit_bias=None, chunks: int = ROUTER_CHUNKS) -> np.ndarray:
    xv, wv = _values(x), _values(w_r)
    T, H = xv.shape
    E = wv.shape[1]
    assert H % chunks == 0
    b = None if logit_bias is None else np.ascontiguousarray(_np(logit_bias), np.float32)
    out = np.empty((T, E), np.float32)
    inexact = lib().orc_router_logits(_ptr(xv), _ptr(wv), _ptr(b), T, H, E, chunks, _ptr(out))
    assert inexact == 0, "product not exact in fp32"
    return out


def _f32(a):
    return np.ascontiguousarray(np.asarray(_np(a), np.float32))


def router_softmax_topk(logits, top_k: int, renormalize: bool = True, rsf: float = 1.0):
    l = _f32(logits)
    T, E = l.shape
    ids = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float64)
    lib().orc_router_softmax_topk(_ptr(l), T, E, top_k, int(renormalize), float(rsf), _ptr(ids), _ptr(w))
    return ids, w


def sigmoid_fp32(logits) -> np.ndarray:
    l = _f32(logits)
    out = np.empty(l.shape, np.float32)
    lib().orc_sigmoid_fp32(_ptr(l), _ptr(out), l.size)
    return out.astype(np.float64)


def _hazards(logits, margin_log2):
    l = _f32(logits)
    mask = np.empty(l.shape, np.uint8)
    other = np.empty(l.shape, np.float32)
    lib().orc_sigmoid_hazards(_ptr(l), l.size, margin_log2, _ptr(mask), _ptr(other))
    return mask.astype(bool), other


def sigmoid_fp32_hazard_mask(logits, margin_log2: int = -46) -> np.ndarray:
    return _hazards(logits, margin_log2)[0]


def sigmoid_fp32_hazards(logits, margin_log2: int = -46) -> int:
    return int(np.count_nonzero(sigmoid_fp32_hazard_mask(logits, margin_log2)))


def sigmoid_fp32_other(logits) -> np.ndarray:
    return _hazards(logits, -46)[1].astype(np.float64)


def router_grouped_sigmoid_topk(logits, correction_bias, top_k: int, n_group: int, topk_group: int,
                                renormalize: bool = True, rsf: float = 1.0, scores=None):
    l = _f32(logits)
    T, E = l.shape
    b = None if correction_bias is None else _f32(correction_bias)
    s = None if scores is None else _f32(scores)
    ids = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float64)
    lib().orc_router_grouped_topk(_ptr(l), _ptr(s), _ptr(b), T, E, top_k, n_group, topk_group, int(renormalize),
                                  float(rsf), _ptr(ids), _ptr(w))
    return ids, w


def route(cfg, logits, correction_bias=None):
    if cfg["route"] == "softmax":
        return router_softmax_topk(logits, cfg["top_k"], cfg.get("renormalize", True), cfg["rsf"])
    return router_grouped_sigmoid_topk(logits, correction_bias, cfg["top_k"], cfg["n_group"], cfg["topk_group"],
                                       cfg.get("renormalize", True), cfg["rsf"])


# ------------------------------------------------------------------ sort, gate, expert


def sorted_capacity(T: int, top_k: int, E: int, block_m: int) -> int:
    return int(lib().orc_sorted_capacity(T, top_k, E, block_m))


def align_sort(topk_ids, E: int, block_m: int):
    ids = np.ascontiguousarray(np.asarray(topk_ids, np.int32))
    T, k = ids.shape
    cap = sorted_capacity(T, k, E, block_m)
    srt = np.empty(cap, np.int32)
    be = np.empty(cap // block_m + 1, np.int32)
    cnt = np.empty(E, np.int32)
    off = np.empty(E + 1, np.int32)
    npad = np.zeros(1, np.int32)
    r = lib().orc_align_sort(_ptr(ids), T, k, E, block_m, _ptr(srt), _ptr(be), _ptr(cnt), _ptr(off), _ptr(npad))
    assert r == 0, "expert id out of range"
    n = int(npad[0])
    return {"sorted_ids": srt[:n].copy(), "block_expert": be[: n // block_m].copy(), "expert_counts": cnt,
            "expert_offsets": off, "num_padded": n}


def shared_gate(x, w, apply_sigmoid: bool = True, out_format=BF16) -> np.ndarray:
    xv = _values(x)
    if xv.ndim == 1:
        xv = xv[None, :]
    wv = _values(w)
    T, K = xv.shape
    g = np.empty(T, np.float64)
    lib().orc_shared_gate(_ptr(xv), _ptr(wv), T, K, int(apply_sigmoid), 0 if out_format.name == "bf16" else 1,
                          _ptr(g))
    return g


def _expert(x_t, w13, w2, I, hmode, s_x, s_w13, s_w2):
    x = _f64(x_t)
    a13, a2 = _f64(w13), _f64(w2)
    H = x.size
    assert a13.shape == (2 * I, H) and a2.shape == (H, I)
    y = np.empty(H, np.float64)
    h = np.empty(I, np.float64)
    lib().orc_expert_forward(_ptr(x), _ptr(a13), _ptr(a2), H, I, {"bf16": 0, "fp8": 1, "mxfp8": 2}[hmode],
                             float(s_x), float(s_w13), float(s_w2), _ptr(y), _ptr(h))
    return y, h


def expert_hidden(x_t, w13, I: int, s_x=1.0, s_w13=1.0):
    H = np.asarray(x_t).size
    return _expert(x_t, w13, np.zeros((H, I)), I, "bf16", s_x, s_w13, 1.0)[1]


def expert_forward(x_t, w13, w2, I: int, hmode: str, s_x=1.0, s_w13=1.0, s_w2=1.0):
    return _expert(x_t, w13, w2, I, hmode, s_x, s_w13, s_w2)[0]


def shared_pieces(Is: int, I: int) -> int:
    return -(-Is // I)


# ------------------------------------------------------------------ the layer


def _raw(t, kind):
    """Contiguous numpy array of a stored input: 'u16' bit patterns of bf16
    tensors (float arrays holding bf16 values are converted to their bit
    patterns, exactly), 'u8' codes, 'f64' fp8 scales (as given, widened)."""
    if t is None:
        return None
    a = _np(t)
    if kind == "u16":
        if a.dtype != np.uint16:
            import torch
            v = np.asarray(a, np.float64)
            b = torch.from_numpy(v).to(torch.bfloat16)
            assert np.array_equal(b.double().numpy(), v), "bf16 operand holds values that are not bf16 numbers"
            a = b.view(torch.int16).numpy().view(np.uint16)
    elif kind == "u8":
        a = a.view(np.uint8) if a.dtype != np.uint8 else a
    else:
        a = np.asarray(a, np.float64)
    return np.ascontiguousarray(a)


def _layer_struct(cfg: dict, inp: dict):
    """The OrcLayer of a config and its stored inputs, and the arrays it points
    to (kept alive by the caller)."""
    T, H, E, k, I, Is = (cfg[n] for n in ("T", "H", "E", "top_k", "I", "Is"))
    fmt = cfg["dtype"]
    wk = "u16" if fmt == "bf16" else "u8"
    sk = "f64" if fmt == "fp8" else "u8"
    keep = {
        "logits": _f32(inp["logits"]),
        "corr_bias": None if inp.get("correction_bias") is None else _f32(inp["correction_bias"]),
        "x": _raw(inp["x"], wk),
        "x_scale": _raw(inp.get("x_scale"), sk) if fmt != "bf16" else None,
        "w_gate": _raw(inp.get("w_gate"), "u16") if cfg.get("shared_gate", False) else None,
    }
    for n in ("w13", "w2", "w13s", "w2s"):
        keep[n] = _raw(inp[n], wk)
        keep[n + "_scale"] = _raw(inp.get(n + "_scale"), sk) if fmt != "bf16" else None
    L = OrcLayer()
    L.T, L.H, L.E, L.top_k, L.I, L.Is = T, H, E, k, I, Is
    L.fmt = LAYER_FMT[fmt]
    L.route = 0 if cfg["route"] == "softmax" else 1
    L.n_group, L.topk_group = cfg.get("n_group", 1), cfg.get("topk_group", 1)
    L.renormalize = int(cfg.get("renormalize", True))
    L.rsf = float(cfg["rsf"])
    L.shared_gate = int(cfg.get("shared_gate", False))
    for n, a in keep.items():
        setattr(L, n, _ptr(a))
    return L, keep


def moe_layer(cfg: dict, inp: dict, tokens=None, shared_fused: bool = False, threads: int = 0,
              want_h: bool = False) -> dict:
    """The layer, token by token (see orc_moe_layer in moe_oracle.cpp).
    Same keys in and out as the numpy oracle's ``moe_layer``; ``threads`` = 0
    uses every host thread. ``want_h`` adds the stage-1 values of the
    computed tokens: ``h_raw`` / ``h_q`` [n, k, I] per routed slot (before and
    after quantisation) and ``h_raw_shared`` / ``h_q_shared`` [n, Is]."""
    T, H, k, I, Is = cfg["T"], cfg["H"], cfg["top_k"], cfg["I"], cfg["Is"]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    tok = np.ascontiguousarray(tokens.astype(np.int32))
    L, _keep = _layer_struct(cfg, inp)
    n = len(tok)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    g = np.empty(n, np.float64)
    addend = np.empty((n, H), np.float64)
    routed = np.empty((n, H), np.float64)
    out = np.empty((n, H), np.float64)
    hs = [np.zeros((n, k, I)), np.zeros((n, k, I)), np.zeros((n, Is)), np.zeros((n, Is))] if want_h else [None] * 4
    r = lib().orc_moe_layer_h(ctypes.byref(L), _ptr(tok), n, int(shared_fused), int(threads), _ptr(ids), _ptr(w),
                              _ptr(g), _ptr(addend), _ptr(routed), _ptr(out), *[_ptr(a) for a in hs])
    assert r == 0, "invalid layer arguments"
    res = {"topk_ids": ids, "topk_weights": w, "gate": g, "addend": addend, "routed": routed, "out": out,
           "tokens": tokens}
    if want_h:
        res.update(h_raw=hs[0], h_q=hs[1], h_raw_shared=hs[2], h_q_shared=hs[3])
    return res


class LayerUnits:
    """Expert calls of one layer as separate units of work (the CPU
    reference's timing unit): ``run(units)`` computes, for each (token, slot)
    pair (slot -1: the shared expert), that expert's output on that token, in
    parallel over the host threads. Routing comes from the oracle."""

    def __init__(self, cfg: dict, inp: dict, threads: int = 0):
        self.cfg = cfg
        self.L, self._keep = _layer_struct(cfg, inp)
        self.ids = np.ascontiguousarray(route(cfg, inp["logits"], inp.get("correction_bias"))[0].astype(np.int32))
        self.threads = threads

    def run(self, units):
        u = np.asarray(units, np.int32).reshape(-1, 2)
        ut, uj = np.ascontiguousarray(u[:, 0]), np.ascontiguousarray(u[:, 1])
        y = np.empty((len(u), self.cfg["H"]), np.float64)
        r = lib().orc_layer_units(ctypes.byref(self.L), _ptr(self.ids), _ptr(ut), _ptr(uj), len(u), self.threads,
                                  _ptr(y))
        assert r == 0, "invalid unit"
        return y


def tolerance_ok(out, ref, rel_rms: float):
    """max|out - ref| <= rel_rms * rms(ref) (the stated float tolerance)."""
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = math.sqrt(float(np.mean(ref * ref))) if ref.size else 0.0
    err = float(np.max(np.abs(out - ref))) if ref.size else 0.0
    return err <= rel_rms * rms, err, rms


def num_threads() -> int:
    return int(lib().orc_num_threads())


def _table():
    return e4m3_decode(np.arange(256, dtype=np.uint8))


def __getattr__(name):
    if name == "E4M3_TABLE":
        return _table()
    if name == "E2M1_TABLE":
        return e2m1_decode(np.arange(16, dtype=np.uint8))
    raise AttributeError(name)
