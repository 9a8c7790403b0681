"""Plain CPU oracle of the routed + shared-expert MoE layer forward pass.

TEST INFRASTRUCTURE ONLY. This module is the slow, obviously-correct statement of
what the GPU path computes. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. The
product path (``routed_shared_experts_b200``) never imports it, and it imports
nothing from the product path.

Arithmetic is float64 (numpy), one token / one (token, slot) pair at a time.
Library primitives used as steps: ``numpy`` matrix-vector products, a stable
``argsort`` and ``exp``. Number formats (bf16, fp16, fp8 e4m3, fp4 e2m1, ue8m0
block scales) are implemented here from their definitions, not taken from a
library.

Sources (web pages; section names as printed on them):

* vllm-project/vllm PR 65207 "[ROCm][MoE] accumulate shared-expert output in
  AITER stage 2", section "Purpose", commit 1 (routed_scaling_factor folded into
  the top-k weights of ``biased_grouped_topk``) and commit 2 (the shared-expert
  output is the stage-2 addend, accumulated in the GEMM2 epilogue instead of a
  separate bf16 add); reviewer measurements ("Commits 2 and 3": ``moe_sorting``
  without zeroing).
* ROCm/aiter PR 6106 "[Triton/Gluon] Add per token scale to a8w8 moe gemm",
  section "Technical Details": per-row activation scale and per-expert weight
  scale multiply the fp32 accumulator before activation and fused quant; rows
  follow the gather index; MXFP8 uses BLOCK_K = 32 with K % 32 == 0.
* vllm-project/vllm PR 56789 (shared_expert_gate as a tiny dot), sections
  "Summary" and "Commits": ``sigmoid(shared_expert_gate(x))`` computed as one
  fp32-accumulated dot with the sigmoid folded in, output stored in the input
  dtype so that the store does the rounding.
* vllm-project/vllm PR 61503 "Fused heterogeneous MoE", section "Overview":
  routed experts plus a shared expert in one MoE layer.

Where the pages leave a step open the reading taken is stated beside the code
(softmax/grouped-sigmoid tie rules, sort layout, quantisation points, MX rule).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# ---------------------------------------------------------------------------
# Number formats, written from their definitions.
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class FloatFormat:
    """A binary floating-point format: ``p`` significant bits (implicit bit
    included), smallest normal exponent ``emin``, largest finite value
    ``max_finite``; ``saturate`` clamps overflow to ``max_finite`` (the
    ``satfinite`` conversion), otherwise overflow becomes infinity."""

    name: str
    p: int
    emin: int
    max_finite: float
    saturate: bool


BF16 = FloatFormat("bf16", 8, -126, float((2 - 2.0**-7) * 2.0**127), False)
FP16 = FloatFormat("fp16", 11, -14, 65504.0, False)
FP32 = FloatFormat("fp32", 24, -126, float((2 - 2.0**-23) * 2.0**127), False)
# OCP 8-bit "E4M3" (the "fn" variant: no infinities, a single NaN pattern
# S.1111.111 per sign), bias 7: largest finite 1.75 * 2**8 = 448.
E4M3 = FloatFormat("e4m3", 4, -6, 448.0, True)
E4M3_MAX = 448.0


def round_to_format(x, fmt: FloatFormat) -> np.ndarray:
    """Round float64 values to the nearest value of ``fmt`` (ties to even).

    With x = m * 2**e (0.5 <= |m| < 1) the binade exponent is e-1; the spacing
    of representable values there is 2**(max(e-1, emin) - (p-1)) (the lower
    bound gives the subnormal spacing). ``np.rint`` rounds half to even, which
    is exactly round-to-nearest-even on the scaled value.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    binade = np.maximum(e.astype(np.int64) - 1, fmt.emin)
    quantum = np.ldexp(1.0, (binade - (fmt.p - 1)).astype(np.int32))
    q = np.rint(x / quantum) * quantum
    over = np.abs(q) > fmt.max_finite
    if fmt.saturate:
        q = np.where(over, np.copysign(fmt.max_finite, q), q)
    else:
        q = np.where(over, np.copysign(np.inf, q), q)
    return np.where(x == 0, x, q)


def bf16_round(x) -> np.ndarray:
    return round_to_format(x, BF16)


def fp16_round(x) -> np.ndarray:
    return round_to_format(x, FP16)


def fp32_round(x) -> np.ndarray:
    return round_to_format(x, FP32)


def _e4m3_value(c: int) -> float:
    """Value of one OCP E4M3 (fn) byte: sign bit, 4 exponent bits (bias 7),
    3 mantissa bits; exponent field 0 is subnormal (m/8 * 2**-6); the pattern
    S.1111.111 is NaN (there is no infinity)."""
    sign = -1.0 if c & 0x80 else 1.0
    ef = (c >> 3) & 0xF
    mf = c & 0x7
    if ef == 15 and mf == 7:
        return math.nan
    if ef == 0:
        return sign * (mf / 8.0) * 2.0**-6
    return sign * (1.0 + mf / 8.0) * 2.0 ** (ef - 7)


E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], np.float64)


def e4m3_decode(codes) -> np.ndarray:
    """Decode e4m3 bytes through the 256-entry table of ``_e4m3_value``."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def _e2m1_value(c: int) -> float:
    """Value of one OCP E2M1 (FP4) code, bits 0-3 of ``c``: sign bit 3, two
    exponent bits (bias 1), one mantissa bit; exponent field 0 is subnormal
    (m/2 * 2**0). Every pattern is a finite number (largest 6, no NaN)."""
    sign = -1.0 if c & 0x8 else 1.0
    ef = (c >> 1) & 0x3
    mf = c & 0x1
    if ef == 0:
        return sign * (mf / 2.0)
    return sign * (1.0 + mf / 2.0) * 2.0 ** (ef - 1)


E2M1_TABLE = np.array([_e2m1_value(c) for c in range(16)], np.float64)


def e2m1_unpack(packed) -> np.ndarray:
    """Codes [..., 2n] of e2m1 values stored two per byte [..., n]: element 2j
    in bits 0-3 of byte j, element 2j+1 in bits 4-7 (the storage order of the
    MXFP4 weights)."""
    b = np.asarray(packed, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def e2m1_decode(codes) -> np.ndarray:
    """Decode e2m1 codes (one per byte, bits 0-3) through ``_e2m1_value``."""
    return E2M1_TABLE[np.asarray(codes, dtype=np.uint8) & 0xF]


def bf16_bits_decode(bits) -> np.ndarray:
    """bf16 is the upper half of an IEEE binary32: widen the 16-bit pattern."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def fp16_bits_decode(bits) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def ue8m0_decode(scale_bytes) -> np.ndarray:
    """An MX block scale byte b stands for 2**(b - 127) (byte 255 is NaN; it is
    never produced here)."""
    b = np.asarray(scale_bytes, dtype=np.uint8).astype(np.int64)
    return np.ldexp(1.0, (b - 127).astype(np.int32))


def mx_block_exponent(amax) -> np.ndarray:
    """Shared exponent of one 32-element MX block for E4M3 elements.

    Reading (OCP MX v1.0 conversion rule): X = floor(log2(amax)) - emax_elem
    with emax_elem = 8 for E4M3, clamped to the ue8m0 range [-127, 127]; an
    all-zero block takes X = -127 (byte 0). floor(log2) is taken exactly from
    the binary exponent (frexp), not from a rounded logarithm.
    """
    a = np.asarray(amax, dtype=np.float64)
    _, e = np.frexp(a)
    x = e.astype(np.int64) - 1 - 8
    x = np.clip(x, -127, 127)
    return np.where(a == 0, -127, x)


def e4m3_encode(values) -> np.ndarray:
    """Codes (uint8) of values that are already e4m3 numbers (finite, |v| <= 448):
    the inverse of e4m3_decode. E4M3 is sign-magnitude, so the sign bit comes
    from the value's sign, zero included: a negative value that rounded to zero
    (-0.0) encodes as 0x80, as the OCP format defines -0."""
    v = np.asarray(values, np.float64)
    mag = np.abs(v)
    table_v = E4M3_TABLE[:0x7F]  # codes 0x00..0x7E: the non-negative values, increasing
    idx = np.clip(np.searchsorted(table_v, mag), 0, 0x7E)
    assert np.array_equal(table_v[idx], mag), "not an e4m3 value"
    return (idx | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def quantize_activations(x, mode: str):
    """Quantisation of the layer's bf16 activations x [T, H] to the stage-1
    operand formats (ROCm/aiter PR 6106, "Technical Details": per-token
    activation scales; MXFP8 with BLOCK_K = 32). Returns (codes uint8 [T, H],
    scales): fp32 [T] for 'fp8', ue8m0 bytes [T, H/32] for 'mxfp8'.

    'fp8': s = fp32(amax / 448) per row (amax = 0 gives s = 1); each code is
    e4m3_rn(fp32(x / s)) with saturation - the quotient rounded to fp32 first,
    the precision the kernel decides in, then to e4m3.
    'mxfp8': per 32 columns X = mx_block_exponent(amax), byte X + 127, codes
    e4m3_rn(x * 2^-X) (exact scaling, then one rounding).
    """
    x = np.asarray(x, np.float64)
    T, H = x.shape
    if mode == "fp8":
        amax = np.max(np.abs(x), axis=1)
        s = np.where(amax > 0, fp32_round(amax / E4M3_MAX), 1.0)
        q = fp32_round(x.astype(np.float32) / s.astype(np.float32)[:, None])
        vals = round_to_format(q, E4M3)
        return e4m3_encode(vals), s.astype(np.float32)
    if mode == "mxfp8":
        assert H % 32 == 0
        blk = x.reshape(T, H // 32, 32)
        X = mx_block_exponent(np.max(np.abs(blk), axis=-1))
        vals = round_to_format(blk * np.ldexp(1.0, -X.astype(np.int32))[..., None], E4M3)
        return e4m3_encode(vals.reshape(T, H)), (X + 127).astype(np.uint8)
    raise ValueError(mode)


# ---------------------------------------------------------------------------
# Router (top-k). vllm PR 65207, "Purpose", commit 1: routed_scaling_factor is
# folded into the top-k weights inside the top-k kernel.
# ---------------------------------------------------------------------------


def _desc_order(keys: np.ndarray) -> np.ndarray:
    """Indices sorted by (key descending, index ascending): a stable sort of the
    negated keys keeps equal keys in index order, so ties go to the lower index.
    Negating a float is exact."""
    return np.argsort(-keys, axis=-1, kind="stable")


ROUTER_CHUNKS = 8


def router_logits(x, w_r, logit_bias=None, chunks: int = ROUTER_CHUNKS) -> np.ndarray:
    """Router logits ``x . W_r`` in one fixed fp32 order (float32 result [T, E]).

    The pages give no arithmetic for the router linear (vllm-project/vllm
    PR 65207, "Purpose", passes the gating output to ``biased_grouped_topk``);
    the fused router of this implementation defines one order, written out here
    so that routing decisions made from these logits can be compared bit for
    bit: with ``c = H / chunks``, for each chunk j the fp32 running sum
    ``p_j = (...((x_{jc} w_{jc}) + x_{jc+1} w_{jc+1}) + ...)`` in index order,
    then ``logit = (...((p_0 + p_1) + p_2) + ...) + p_{chunks-1}``, then
    ``+ logit_bias[e]`` (fp32) when given. Every addition rounds to nearest
    fp32. The products of bf16 or fp16 inputs are exact in fp32 (at most
    8 + 8 or 11 + 11 significant bits), so only the additions round; this is
    asserted for the inputs given.

    x: [T, H] values of a bf16/fp16 tensor; w_r: [H, E] of the same format.
    """
    x = np.asarray(x, np.float64)
    w = np.asarray(w_r, np.float64)
    T, H = x.shape
    H2, E = w.shape
    assert H == H2 and H % chunks == 0
    c = H // chunks
    out = None
    for j in range(chunks):
        acc = np.zeros((T, E), np.float32)
        for h in range(j * c, (j + 1) * c):
            prod = np.outer(x[:, h], w[h, :])
            p32 = prod.astype(np.float32)
            assert np.array_equal(p32.astype(np.float64), prod), "product not exact in fp32"
            acc = acc + p32
        out = acc if out is None else out + acc
    if logit_bias is not None:
        out = out + np.asarray(logit_bias, np.float32)[None, :]
    return out


def router_softmax_topk(logits, top_k: int, renormalize: bool = True, rsf: float = 1.0):
    """Softmax top-k.

    Selection: softmax is strictly increasing in the logit, so the k largest
    probabilities are the k largest logits; they are picked on the fp32 logits
    with ties to the lower expert index. Weights (float64):
    renormalize -> exp(l_j - m) / sum_sel exp(l_i - m) * rsf (m = largest selected
    logit); otherwise softmax over all E, taken at the selected experts, * rsf.
    Returns (ids int32 [T,k] in selection order, weights float64 [T,k]).
    """
    l = np.asarray(logits, dtype=np.float32).astype(np.float64)
    T, E = l.shape
    ids = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float64)
    for t in range(T):
        sel = _desc_order(l[t])[:top_k]
        ids[t] = sel
        if renormalize:
            p = np.exp(l[t, sel] - l[t, sel[0]])
            w[t] = p / p.sum() * rsf
        else:
            p_all = np.exp(l[t] - l[t].max())
            w[t] = p_all[sel] / p_all.sum() * rsf
    return ids, w


def sigmoid_fp32(logits) -> np.ndarray:
    """Router score s = sigmoid(l) evaluated in float64 and rounded once to fp32
    (the reading that makes the selection reproducible across machines)."""
    l = np.asarray(logits, dtype=np.float32).astype(np.float64)
    return fp32_round(1.0 / (1.0 + np.exp(-l)))


def sigmoid_fp32_hazard_mask(logits, margin_log2: int = -46) -> np.ndarray:
    """Scores whose float64 sigmoid lies within 2**margin_log2 (relative) of an
    fp32 rounding midpoint. Two correct evaluations of 1/(1+exp(-l)) in float64
    (exp within a few ulps, then one add and one divide) differ by well under
    2**-48 relative, so only these scores can round to different fp32 values
    on two machines."""
    l = np.asarray(logits, dtype=np.float32).astype(np.float64)
    v = 1.0 / (1.0 + np.exp(-l))
    r = fp32_round(v)
    _, e = np.frexp(r)
    half_ulp = np.ldexp(1.0, (e.astype(np.int64) - 1 - 24).astype(np.int32))
    mid = np.where(v >= r, r + half_ulp, r - half_ulp)
    return np.abs(v - mid) < np.abs(v) * 2.0**margin_log2


def sigmoid_fp32_hazards(logits, margin_log2: int = -46) -> int:
    """Number of scores flagged by ``sigmoid_fp32_hazard_mask``."""
    return int(np.count_nonzero(sigmoid_fp32_hazard_mask(logits, margin_log2)))


def sigmoid_fp32_other(logits) -> np.ndarray:
    """The fp32 neighbour of the float64 sigmoid on the other side of it from
    ``sigmoid_fp32`` (the rounding another machine may take at a hazard)."""
    l = np.asarray(logits, dtype=np.float32).astype(np.float64)
    v = 1.0 / (1.0 + np.exp(-l))
    r = sigmoid_fp32(logits).astype(np.float32)
    up = np.nextafter(r, np.float32(np.inf))
    dn = np.nextafter(r, np.float32(-np.inf))
    return np.where(v >= r.astype(np.float64), up, dn).astype(np.float64)


def router_grouped_sigmoid_topk(
    logits,
    correction_bias,
    top_k: int,
    n_group: int,
    topk_group: int,
    renormalize: bool = True,
    rsf: float = 1.0,
    scores=None,
):
    """Biased grouped sigmoid top-k (the ``biased_grouped_topk`` of vllm PR
    65207, "Purpose", commit 1), with the usual reading of its steps:

    1. s_e = sigmoid(l_e) as fp32 (``sigmoid_fp32``);
    2. choice key c_e = fp32(s_e + b_e) (b = correction bias, 0 if absent);
    3. group score = fp32 sum of the two largest c in the group (the single c
       when a group holds one expert);
    4. keep the ``topk_group`` groups of highest score (ties: lower group);
    5. among experts of kept groups pick k by (c desc, index asc);
    6. weights use the unbiased scores: s_j / sum_sel s * rsf (renormalize) or
       s_j * rsf — the scale is applied here, inside top-k.
    ``scores`` replaces step 1 with given fp32 scores (used to evaluate the
    other rounding of a hazard score).
    """
    l = np.asarray(logits, dtype=np.float32)
    T, E = l.shape
    gsize = E // n_group
    s = (sigmoid_fp32(l) if scores is None else np.asarray(scores, np.float64)).astype(np.float32)
    b = np.zeros(E, np.float32) if correction_bias is None else np.asarray(correction_bias, np.float32)
    c = (s + b[None, :]).astype(np.float32)  # IEEE fp32 addition
    ids = np.empty((T, top_k), np.int32)
    w = np.empty((T, top_k), np.float64)
    for t in range(T):
        groups = c[t].reshape(n_group, gsize)
        if gsize == 1:
            score = groups[:, 0].copy()
        else:
            top2 = -np.sort(-groups, axis=1)[:, :2]
            score = (top2[:, 0] + top2[:, 1]).astype(np.float32)  # fp32 add
        kept = _desc_order(score.astype(np.float64))[:topk_group]
        allowed = np.zeros(E, bool)
        for g in kept:
            allowed[g * gsize:(g + 1) * gsize] = True
        key = np.where(allowed, c[t].astype(np.float64), -np.inf)
        sel = _desc_order(key)[:top_k]
        ids[t] = sel
        s_sel = s[t, sel].astype(np.float64)
        w[t] = (s_sel / s_sel.sum() if renormalize else s_sel) * rsf
    return ids, w


# ---------------------------------------------------------------------------
# Align / sort by expert. vllm PR 65207 reviewer measurements, "Commits 2 and
# 3": moe_sorting runs without zeroing the output; ROCm/aiter PR 6106
# "Technical Details": rows of the grouped GEMM follow a gather index.
# ---------------------------------------------------------------------------


def sorted_capacity(T: int, top_k: int, E: int, block_m: int) -> int:
    """Upper bound of the padded sorted length: every expert may add up to
    block_m - 1 padding slots."""
    return T * top_k + E * (block_m - 1)


def align_sort(topk_ids, E: int, block_m: int):
    """Stable counting sort of the flat slots f = t*k + j by expert.

    Reading: segments in expert order 0..E-1; inside a segment ascending f;
    each segment padded to a multiple of block_m with the sentinel T*k (an
    expert with no slot gets no block); expert_offsets = exclusive prefix sum of
    the padded sizes; block_expert[b] = owner of block b; num_padded =
    expert_offsets[E]. Returns a dict of int32 arrays; sorted_ids has length
    num_padded (entries past it are not part of the result).
    """
    ids = np.asarray(topk_ids, dtype=np.int64)
    T, k = ids.shape
    flat = ids.reshape(-1)
    sentinel = T * k
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    segments = []
    blocks = []
    for e in range(E):
        rows = np.nonzero(flat == e)[0]  # ascending flat index: stable
        counts[e] = rows.size
        padded = -(-rows.size // block_m) * block_m
        seg = np.full(padded, sentinel, np.int64)
        seg[: rows.size] = rows
        segments.append(seg)
        blocks.extend([e] * (padded // block_m))
        offsets[e + 1] = offsets[e] + padded
    sorted_ids = np.concatenate(segments).astype(np.int32) if segments else np.zeros(0, np.int32)
    return {
        "sorted_ids": sorted_ids,
        "block_expert": np.asarray(blocks, np.int32),
        "expert_counts": counts,
        "expert_offsets": offsets,
        "num_padded": int(offsets[E]),
    }


# ---------------------------------------------------------------------------
# Shared-expert gate. vllm PR 56789, "Summary" and "Commits": sigmoid of a
# 1 x K dot, fp32 accumulation, stored in the input dtype (the store rounds).
# ---------------------------------------------------------------------------


def shared_gate(x, w, apply_sigmoid: bool = True, out_format: FloatFormat = BF16) -> np.ndarray:
    """g_t = round_to(dtype of x)( sigmoid(sum_h x[t,h] * w[h]) ), the dot and
    the sigmoid in float64, one rounding at the store."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    d = x @ w
    v = 1.0 / (1.0 + np.exp(-d)) if apply_sigmoid else d
    return round_to_format(v, out_format)


# ---------------------------------------------------------------------------
# Expert MLP and quantisation of the intermediate h.
# ---------------------------------------------------------------------------


def silu(z):
    """z * sigmoid(z) = z / (1 + exp(-z)); for very negative z exp(-z)
    overflows to inf and the quotient is the correct limit, -0."""
    z = np.asarray(z, np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def quantize_h(h, mode: str) -> np.ndarray:
    """Quantisation point of the stage-1 output, returning the dequantised
    float64 values that stage 2 multiplies.

    * 'bf16': h is stored as bf16.
    * 'fp8': one fp32 scale per row, s = fp32(amax / 448); q = e4m3_rn(h / s)
      with saturation; value q * s (ROCm/aiter PR 6106 "Technical Details":
      "fused quant" in the epilogue, per-row scales). amax = 0 gives s = 1, q = 0.
    * 'mxfp8': per 32 consecutive columns, X = mx_block_exponent(amax);
      q = e4m3_rn(h * 2**-X); value q * 2**X (BLOCK_K = 32, K % 32 == 0).
    """
    h = np.asarray(h, np.float64)
    if mode == "bf16":
        return bf16_round(h)
    if mode == "fp8":
        amax = np.max(np.abs(h), axis=-1, keepdims=True)
        s = np.where(amax > 0, fp32_round(amax / E4M3_MAX), 1.0)
        q = round_to_format(h / s, E4M3)
        return q * s
    if mode == "mxfp8":
        n = h.shape[-1]
        assert n % 32 == 0
        blk = h.reshape(h.shape[:-1] + (n // 32, 32))
        X = mx_block_exponent(np.max(np.abs(blk), axis=-1, keepdims=True))
        scale = np.ldexp(1.0, X.astype(np.int32))
        q = round_to_format(blk / scale, E4M3)
        return (q * scale).reshape(h.shape)
    raise ValueError(mode)


def expert_hidden(x_t, w13, I: int, s_x=1.0, s_w13=1.0):
    """Stage-1 value of one expert on one token, before quantisation:
    acc1 = W13 @ x (2I outputs); a = acc1 * s_x * s_w13 (scales on the fp32
    accumulator before the activation); h = SiLU(a[:I]) * a[I:]."""
    acc1 = np.asarray(w13, np.float64) @ np.asarray(x_t, np.float64)
    a = acc1 * s_x * s_w13
    return silu(a[:I]) * a[I:]


def expert_forward(x_t, w13, w2, I: int, hmode: str, s_x=1.0, s_w13=1.0, s_w2=1.0):
    """One expert on one token (float64), in the order the pages give:
    h = ``expert_hidden``; h is quantised (``quantize_h``); y = (W2 @ h) * s_w2,
    where a per-row scale of h is already inside the dequantised h. MX block
    scales are inside the decoded operands. Returns y [H].
    """
    hq = quantize_h(expert_hidden(x_t, w13, I, s_x, s_w13), hmode)
    return (np.asarray(w2, np.float64) @ hq) * s_w2


# ---------------------------------------------------------------------------
# The layer.
# ---------------------------------------------------------------------------


def decode_operand(t, fmt: str, scale=None):
    """Float64 values of a stored operand. fmt: 'bf16' / 'fp16' (uint16 bit
    patterns or torch tensors of that dtype), 'fp8' (uint8 e4m3 codes; a
    per-tensor or per-row scale is applied by the caller, after the matmul),
    'mxfp8' (uint8 codes with ue8m0 bytes per 32 columns in ``scale``), or
    'mxfp4' (e2m1 codes two per byte, ``e2m1_unpack``, with ue8m0 bytes per 32
    unpacked columns in ``scale``)."""
    a = _as_numpy(t)
    if fmt == "mxfp4":
        v = e2m1_decode(e2m1_unpack(a))
        sc = ue8m0_decode(_as_numpy(scale))
        n = v.shape[-1]
        return (v.reshape(v.shape[:-1] + (n // 32, 32)) * sc[..., None]).reshape(v.shape)
    if fmt in ("bf16", "fp16"):
        if a.dtype == np.uint16:
            return bf16_bits_decode(a) if fmt == "bf16" else fp16_bits_decode(a)
        return a.astype(np.float64)
    if fmt == "fp8":
        return e4m3_decode(a)
    if fmt == "mxfp8":
        v = e4m3_decode(a)
        sc = ue8m0_decode(_as_numpy(scale))
        n = v.shape[-1]
        return (v.reshape(v.shape[:-1] + (n // 32, 32)) * sc[..., None]).reshape(v.shape)
    raise ValueError(fmt)


def _as_numpy(t):
    """Accept numpy arrays or CPU torch tensors; bf16/fp16 tensors are widened
    (exactly) to float64, fp8 byte tensors are returned as uint8 codes."""
    if isinstance(t, np.ndarray):
        return t
    try:
        import torch
    except ImportError:  # pragma: no cover
        return np.asarray(t)
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu()
        if t.dtype in (torch.bfloat16, torch.float16):
            return t.to(torch.float64).numpy()
        return t.numpy()
    return np.asarray(t)


def route(cfg, logits, correction_bias=None):
    """Top-k routing of every token, per the config's mode."""
    if cfg["route"] == "softmax":
        return router_softmax_topk(logits, cfg["top_k"], cfg.get("renormalize", True), cfg["rsf"])
    return router_grouped_sigmoid_topk(
        logits, correction_bias, cfg["top_k"], cfg["n_group"], cfg["topk_group"],
        cfg.get("renormalize", True), cfg["rsf"],
    )


def shared_pieces(Is: int, I: int) -> int:
    """Number m of I-wide virtual experts that hold a shared expert of
    intermediate size Is (the last one zero-padded)."""
    return -(-Is // I)


def moe_layer(cfg: dict, inp: dict, tokens=None, shared_fused: bool = False) -> dict:
    """Forward pass of one routed + shared-expert MoE layer, token by token.

    For each token t (all of them, or the listed ``tokens``):
        ids, w      = route(logits_t)
        g_t         = gate(x_t) if the layer has a shared gate, else 1
        addend_t    = bf16( g_t * SharedExpert(x_t) )
        out_t       = bf16( addend_t + sum_j w_j * Expert_{ids_j}(x_t) )
    (vllm PR 65207 "Purpose": the shared output is the addend of stage 2, so the
    routed sum and the addend meet before the single bf16 rounding; commit 1: the
    routed scaling factor is already inside w.)

    ``cfg`` keys: T H E top_k I Is dtype ('bf16'|'fp8'|'mxfp8'|'mxfp4') route
    ('softmax'|'grouped_sigmoid') n_group topk_group rsf renormalize shared_gate.
    ``inp`` keys: logits [T,E] fp32, x, w13 [E,2I,H], w2 [E,H,I], w13s [2Is,H],
    w2s [H,Is], optional correction_bias [E], w_gate [H]; fp8 configs add
    x_scale [T], w13_scale [E], w2_scale [E], w13s_scale [1], w2s_scale [1];
    mxfp8 configs add x_scale [T,H/32], w13_scale [E,2I,H/32], w2_scale
    [E,H,I/32], w13s_scale [2Is,H/32], w2s_scale [H,Is/32] (ue8m0 bytes).
    mxfp4 configs hold the four weight matrices as e2m1 codes two per byte
    (K halved in the stored shape) with the same scale arrays; x and the
    quantisation of h are those of mxfp8 (reading: the pages run MXFP4 weights,
    vllm PR 65207 commit 3, and fix no activation format).

    ``shared_fused``: the shared expert taken as always-selected routed experts
    (vllm-project/vllm PR 61503 "Fused heterogeneous MoE", "Overview"): it is cut
    into m = ceil(Is / I) virtual experts of I intermediate features (gate rows
    v*I..v*I+I-1 with their up rows and W2 columns, zero-padded past Is), each
    computed like a routed expert (its h quantised on its own I columns) with
    weight g_t, and all contributions meet before the one rounding:
        out_t = bf16( sum_j w_j * Expert_{ids_j}(x_t) + sum_v g_t * Piece_v(x_t) )
    ``addend`` then holds the unrounded shared sum.

    Returns routing for all tokens (ids, weights), and for the computed tokens:
    gate [n], addend [n,H], out [n,H] (float64 values of bf16 numbers) and
    ``tokens``.
    """
    T, H, E, k, I, Is = (cfg[n] for n in ("T", "H", "E", "top_k", "I", "Is"))
    fmt = cfg["dtype"]
    afmt = "mxfp8" if fmt == "mxfp4" else fmt  # activations and h
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    ids, w = route(cfg, _as_numpy(inp["logits"]), None if inp.get("correction_bias") is None
                   else _as_numpy(inp["correction_bias"]))

    x_all = decode_operand(inp["x"], afmt, inp.get("x_scale") if afmt == "mxfp8" else None)
    if fmt == "fp8":
        s_x = _as_numpy(inp["x_scale"]).astype(np.float64).reshape(-1)
    else:
        s_x = np.ones(T)

    # shared gate (bf16 configs only carry one)
    if cfg.get("shared_gate", False):
        g = shared_gate(x_all[tokens], decode_operand(inp["w_gate"], fmt), True,
                        BF16 if fmt == "bf16" else FP16)
    else:
        g = np.ones(len(tokens))

    def weights_of(name, e=None):
        wt = inp[name] if e is None else inp[name][e]
        sc = inp.get(name + "_scale")
        if fmt in ("mxfp8", "mxfp4"):
            return decode_operand(wt, fmt, sc if e is None else sc[e]), 1.0
        if fmt == "fp8":
            s = _as_numpy(sc).astype(np.float64).reshape(-1)
            return decode_operand(wt, fmt), float(s[0] if e is None else s[e])
        return decode_operand(wt, fmt), 1.0

    # shared expert -> addend (or, fused, its unrounded sum over the pieces)
    w13s, s13s = weights_of("w13s")
    w2s, s2s = weights_of("w2s")
    addend = np.empty((len(tokens), H))
    if shared_fused:
        m = shared_pieces(Is, I)
        pieces = []
        for v in range(m):
            lo, hi = v * I, min((v + 1) * I, Is)
            p13 = np.zeros((2 * I, H))
            p13[: hi - lo] = w13s[lo:hi]
            p13[I: I + hi - lo] = w13s[Is + lo: Is + hi]
            p2 = np.zeros((H, I))
            p2[:, : hi - lo] = w2s[:, lo:hi]
            pieces.append((p13, p2))
        for i, t in enumerate(tokens):
            addend[i] = sum(g[i] * expert_forward(x_all[t], p13, p2, I, afmt, s_x[t], s13s, s2s)
                            for p13, p2 in pieces)
    else:
        for i, t in enumerate(tokens):
            ys = expert_forward(x_all[t], w13s, w2s, Is, afmt, s_x[t], s13s, s2s)
            addend[i] = bf16_round(g[i] * ys)

    # routed experts: each (token, slot) pair is an independent expert call;
    # pairs are visited expert by expert only so that each expert's weights are
    # decoded once. The per-token sum below runs over j = 0..k-1.
    contrib = np.zeros((len(tokens), k, H))
    pos = {int(t): i for i, t in enumerate(tokens)}
    for e in np.unique(ids[tokens]):
        w13e, s13e = weights_of("w13", e)
        w2e, s2e = weights_of("w2", e)
        for t in tokens:
            for j in range(k):
                if ids[t, j] == e:
                    y = expert_forward(x_all[t], w13e, w2e, I, afmt, s_x[t], s13e, s2e)
                    contrib[pos[int(t)], j] = w[t, j] * y
    routed = np.zeros((len(tokens), H))
    for j in range(k):
        routed += contrib[:, j]
    out = bf16_round(addend + routed)
    return {"topk_ids": ids, "topk_weights": w, "gate": g, "addend": addend,
            "routed": routed, "out": out, "tokens": tokens}


def tolerance_ok(out, ref, rel_rms: float):
    """max|out - ref| <= rel_rms * rms(ref) (the stated float tolerance)."""
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = math.sqrt(float(np.mean(ref * ref))) if ref.size else 0.0
    err = float(np.max(np.abs(out - ref))) if ref.size else 0.0
    return err <= rel_rms * rms, err, rms
