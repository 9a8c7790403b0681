"""Pins of the CPU oracle against things other than itself: closed forms, brute
force on tiny inputs, library special cases and invariants. CPU only.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
swapped operand, a wrong sign or index, a wrong tie rule) fails it.

Every pin runs twice: against the oracle of record, the plain C++ one
(oracle/moe_oracle.cpp through oracle/cpp.py), and against the independent
float64 numpy statement of the same definitions (oracle/moe_oracle.py).
"""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import cpp as _cpp_oracle
from oracle import moe_oracle as _np_oracle

oracle = mo = _cpp_oracle  # set per test by the fixture below
IMPLS = {"cpp": _cpp_oracle, "numpy": _np_oracle}


@pytest.fixture(autouse=True, params=sorted(IMPLS))
def oracle_impl(request):
    """Runs the test against each oracle implementation (module globals
    ``oracle`` and ``mo`` name the one under test)."""
    global oracle, mo
    oracle = mo = IMPLS[request.param]
    yield request.param

# ---------------------------------------------------------------- formats


def test_e4m3_table_matches_closed_form_landmarks():
    # OCP E4M3 landmarks: max normal 0x7E = 448, min normal 0x08 = 2^-6,
    # min subnormal 0x01 = 2^-9, one = 0x38, NaN = 0x7F / 0xFF, -0 = 0x80.
    t = mo.E4M3_TABLE
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x08] == 2.0**-6 and t[0x01] == 2.0**-9 and t[0x38] == 1.0
    assert math.isnan(t[0x7F]) and math.isnan(t[0xFF])
    assert t[0x80] == 0.0 and math.copysign(1, t[0x80]) == -1
    assert t[0x07] == 7 * 2.0**-9 and t[0x0F] == 1.875 * 2.0**-6


def test_ue8m0_decode_is_a_power_of_two_per_byte():
    # OCP MX E8M0 scale: byte b stands for 2^(b - 127); 127 is 1.0
    b = np.arange(255, dtype=np.uint8)
    v = mo.ue8m0_decode(b)
    assert v[127] == 1.0 and v[128] == 2.0 and v[126] == 0.5
    assert v[0] == 2.0**-127 and v[254] == 2.0**127
    assert np.all(v[1:] / v[:-1] == 2.0)


def test_sorted_capacity_bounds_every_padded_sort():
    # T*k slots plus at most block_m - 1 padding rows for each of E experts;
    # a sort where every expert holds one slot reaches the bound exactly
    for T, k, E, bm in ((5, 3, 7, 64), (32, 8, 128, 16), (1, 1, 1, 16), (3, 2, 6, 16)):
        assert oracle.sorted_capacity(T, k, E, bm) == T * k + E * (bm - 1)
    ids = np.arange(6, dtype=np.int64).reshape(3, 2)  # 6 experts, one slot each
    r = oracle.align_sort(ids, 6, 16)
    assert r["num_padded"] == 6 * 16 == oracle.sorted_capacity(3, 2, 6, 16)


def test_e4m3_table_matches_torch_float8_for_all_codes():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = mo.e4m3_decode(np.arange(256))
    both_nan = np.isnan(ref) & np.isnan(ours)
    assert np.all(both_nan | (ref == ours))


def test_e2m1_table_matches_closed_form_landmarks():
    # OCP MX FP4 E2M1: max normal 0b0111 = 6, min normal 0b0010 = 1, the one
    # subnormal 0b0001 = 0.5, -0 = 0b1000; no NaN or infinity.
    t = mo.E2M1_TABLE
    assert t[0b0111] == 6.0 and t[0b1111] == -6.0
    assert t[0b0010] == 1.0 and t[0b0001] == 0.5 and t[0b0000] == 0.0
    assert t[0b1000] == 0.0 and math.copysign(1, t[0b1000]) == -1
    assert list(t[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.all(np.isfinite(t))


def test_e2m1_table_matches_ml_dtypes_for_all_codes():
    ml_dtypes = pytest.importorskip("ml_dtypes")
    ref = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = mo.e2m1_decode(np.arange(16))
    assert np.array_equal(ref, ours)
    assert np.array_equal(np.signbit(ref), np.signbit(ours))


def test_e2m1_unpack_puts_element_2j_in_the_low_nibble():
    assert list(mo.e2m1_unpack(np.array([0x21], np.uint8))) == [1, 2]
    assert list(mo.e2m1_unpack(np.array([0xF7, 0x08], np.uint8))) == [7, 15, 8, 0]
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, (5, 64)).astype(np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    assert np.array_equal(mo.e2m1_unpack(packed), codes)


def test_mxfp4_decode_equals_a_scalar_loop():
    ml_dtypes = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(4)
    rows, K = 3, 96
    packed = rng.integers(0, 256, (rows, K // 2)).astype(np.uint8)
    sc = rng.integers(100, 140, (rows, K // 32)).astype(np.uint8)
    got = mo.decode_operand(packed, "mxfp4", sc)
    for r in range(rows):
        for j in range(K):
            byte = int(packed[r, j // 2])
            code = (byte >> 4) if j % 2 else (byte & 0xF)
            v = float(np.array([code], np.uint8).view(ml_dtypes.float4_e2m1fn)[0])
            assert got[r, j] == v * 2.0 ** (int(sc[r, j // 32]) - 127)


def test_mxfp4_layer_equals_the_mxfp8_layer_on_the_same_values():
    # every e2m1 value is an e4m3 value, so MXFP4 weights re-encoded as e4m3
    # codes (torch's cast) with the same block scales give the same layer
    T, H, E, k, I, Is = 6, 64, 4, 2, 32, 32
    cfg = {"T": T, "H": H, "E": E, "top_k": k, "I": I, "Is": Is, "dtype": "mxfp4", "route": "softmax",
           "n_group": 1, "topk_group": 1, "rsf": 1.0, "renormalize": True, "shared_gate": False}
    g = torch.Generator().manual_seed(5)

    def w4(*shape):
        return torch.randint(0, 256, shape[:-1] + (shape[-1] // 2,), generator=g, dtype=torch.uint8)

    def sc(*shape):
        return torch.randint(118, 124, shape[:-1] + (shape[-1] // 32,), generator=g, dtype=torch.uint8)
    x = torch.randn(T, H, generator=g)
    xq = (x * 8).to(torch.float8_e4m3fn).view(torch.uint8)
    inp = {"logits": torch.randn(T, E, generator=g), "x": xq, "x_scale": torch.full((T, H // 32), 124, dtype=torch.uint8),
           "w13": w4(E, 2 * I, H), "w13_scale": sc(E, 2 * I, H), "w2": w4(E, H, I), "w2_scale": sc(E, H, I),
           "w13s": w4(2 * Is, H), "w13s_scale": sc(2 * Is, H), "w2s": w4(H, Is), "w2s_scale": sc(H, Is),
           "correction_bias": None}
    r4 = oracle.moe_layer(cfg, inp)
    e2m1 = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])

    def as_e4m3(packed):
        lo, hi = packed & 0xF, packed >> 4
        vals = torch.stack([e2m1[lo.long()], e2m1[hi.long()]], dim=-1).reshape(packed.shape[:-1] + (-1,))
        return vals.to(torch.float8_e4m3fn).view(torch.uint8)
    inp8 = dict(inp, **{n: as_e4m3(inp[n]) for n in ("w13", "w2", "w13s", "w2s")})
    r8 = oracle.moe_layer(dict(cfg, dtype="mxfp8"), inp8)
    assert np.array_equal(r4["out"], r8["out"]) and np.array_equal(r4["addend"], r8["addend"])
    assert np.any(r4["out"] != 0)


def test_e4m3_rounding_matches_torch_cast_inside_range():
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.normal(0, 1, 20000) * 10.0 ** rng.uniform(-4, 2.6, 20000),
                        mo.E4M3_TABLE[:126] + 1e-12, (mo.E4M3_TABLE[1:126] + mo.E4M3_TABLE[:125]) / 2])
    v = v[np.abs(v) <= 448]
    ours = oracle.round_to_format(v, oracle.E4M3)
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    # torch rounds from fp32; compare on inputs that are exact in fp32
    exact32 = v.astype(np.float32).astype(np.float64) == v
    assert np.array_equal(ours[exact32], ref[exact32])


def test_e4m3_rounding_at_every_midpoint_and_its_fp32_neighbours():
    # For every pair of adjacent non-negative e4m3 values: the midpoint (a tie),
    # the fp32 numbers just below and just above it, both values, and the fp32
    # numbers next to them; both signs. A misplaced rounding bit, a wrong tie
    # rule or a wrong subnormal spacing changes one of these decisions.
    t = mo.E4M3_TABLE[:0x7F]  # 0 .. 448, increasing
    mid = ((t[1:] + t[:-1]) / 2).astype(np.float32)
    pts = [mid, t.astype(np.float32)]
    for base in (mid, t.astype(np.float32)):
        pts.append(np.nextafter(base, np.float32(np.inf)))
        pts.append(np.nextafter(base, np.float32(-np.inf)))
    v = np.concatenate(pts)
    v = v[(v >= 0) & (v <= 448)]
    v = np.concatenate([v, -v]).astype(np.float32)
    ours = oracle.round_to_format(v.astype(np.float64), oracle.E4M3)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)
    assert np.array_equal(np.signbit(ours[ours == 0]), np.signbit(ref[ref == 0]))


def test_e4m3_ties_to_even_and_saturation():
    # 1.0625 lies midway between 1.0 (mantissa 000) and 1.125 (001): even -> 1.0
    # 1.1875 midway between 1.125 (001) and 1.25 (010): even -> 1.25
    r = oracle.round_to_format(np.array([1.0625, 1.1875, 449.0, 1e9, -500.0, 2.0**-10, 3 * 2.0**-10, 3 * 2.0**-11]),
                               oracle.E4M3)
    assert list(r[:5]) == [1.0, 1.25, 448.0, 448.0, -448.0]
    assert r[5] == 0.0            # half of min subnormal -> ties to even (0)
    assert r[6] == 2.0**-9 * 2    # 1.5 min-subnormal -> even (2)
    assert r[7] == 2.0**-9        # 0.75 min-subnormal -> nearest (1)


def test_bf16_and_fp16_rounding_match_torch_from_fp32():
    rng = np.random.default_rng(3)
    v = (rng.normal(0, 1, 50000) * 10.0 ** rng.uniform(-30, 30, 50000)).astype(np.float32)
    v = np.concatenate([v, np.float32([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8)])])
    v64 = v.astype(np.float64)
    ref_b = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.bf16_round(v64), ref_b)
    vs = v[np.abs(v) < 60000]
    ref_h = torch.from_numpy(vs).to(torch.float16).to(torch.float64).numpy()
    assert np.array_equal(mo.fp16_round(vs.astype(np.float64)), ref_h)
    # ties to even: 1 + 2^-8 -> 1.0 ; 1 + 3*2^-8 -> 1 + 2^-6
    assert oracle.bf16_round(np.array([1 + 2**-8]))[0] == 1.0
    assert oracle.bf16_round(np.array([1 + 3 * 2**-8]))[0] == 1 + 2**-6


def test_fp32_rounding_is_numpy_float32_cast():
    rng = np.random.default_rng(5)
    v = rng.normal(0, 1, 100000) * 10.0 ** rng.uniform(-40, 38, 100000)
    assert np.array_equal(mo.fp32_round(v), v.astype(np.float32).astype(np.float64))


def test_mx_exponent_closed_form_and_shift_invariance():
    # amax in [2^n, 2^(n+1)) -> X = n - 8 ; zero block -> -127
    amax = np.array([1.0, 1.999, 2.0, 448.0, 0.75, 2.0**-130, 0.0, 2.0**200])
    X = oracle.mx_block_exponent(amax)
    assert list(X) == [-8, -8, -7, 0, -9, -127, -127, 127]
    rng = np.random.default_rng(11)
    blk = rng.normal(0, 1, (50, 32))
    q0 = oracle.quantize_h(blk, "mxfp8")
    for n in (-5, 3, 17):
        qn = oracle.quantize_h(blk * 2.0**n, "mxfp8")
        assert np.array_equal(qn, q0 * 2.0**n)   # 2^n scaling moves X by n only


def test_mx_block_max_maps_into_e4m3_range():
    rng = np.random.default_rng(12)
    h = rng.normal(0, 3, (8, 64))
    q = oracle.quantize_h(h, "mxfp8").reshape(8, 2, 32)
    blk = h.reshape(8, 2, 32)
    X = oracle.mx_block_exponent(np.abs(blk).max(-1, keepdims=True))
    codes_vals = q / 2.0**X
    assert np.all(np.abs(codes_vals) <= 448)
    assert np.all(np.isin(np.abs(codes_vals), np.abs(mo.E4M3_TABLE[:127])))


def test_fp8_row_quant_maps_amax_to_448():
    rng = np.random.default_rng(2)
    h = rng.normal(0, 1, (16, 100))
    q = oracle.quantize_h(h, "fp8")
    amax = np.abs(h).max(1, keepdims=True)
    s = mo.fp32_round(amax / 448)
    i = np.abs(h).argmax(1)
    np.testing.assert_allclose(np.abs(q[np.arange(16), i]), 448 * s[:, 0], rtol=0)
    assert np.all(np.isin(np.abs(q / s), np.abs(mo.E4M3_TABLE[:127])))
    assert np.all(oracle.quantize_h(np.zeros((2, 8)), "fp8") == 0)


# ---------------------------------------------------------------- router


def _brute_topk(keys, k):
    """Brute force: the unique k-subset whose every member beats every non-member
    under (key desc, index asc); returned in that order."""
    E = len(keys)
    better = lambda a, b: keys[a] > keys[b] or (keys[a] == keys[b] and a < b)  # noqa: E731
    for sub in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in sub]
        if all(better(a, b) for a in sub for b in rest):
            return sorted(sub, key=lambda e: (-keys[e], e))
    raise AssertionError


# ------------------------------------------------------ activation quantisation


def test_e4m3_encode_inverts_decode():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    assert np.array_equal(oracle.e4m3_encode(mo.e4m3_decode(codes)), codes)
    assert oracle.e4m3_encode(np.array([-0.0]))[0] == 0x80 and oracle.e4m3_encode(np.array([0.0]))[0] == 0


def test_quantize_activations_keeps_the_sign_of_zero_like_torch():
    # a large outlier makes s large, so tiny values round to +-0: negative ones
    # encode as 0x80 in torch's float8_e4m3fn cast as in the oracle
    x = torch.tensor([[300.0, -1e-4, 1e-4, -0.0, 0.0, -3e-4, 5.0, -5.0]]).to(torch.bfloat16)
    codes, s = oracle.quantize_activations(x.double().numpy(), "fp8")
    ref = (x.float() / torch.tensor(s)[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)
    assert codes[0, 1] == 0x80 and codes[0, 2] == 0x00


def test_quantize_activations_fp8_matches_torch_division_and_cast():
    # torch: fp32 division by the fp32 scale, float8_e4m3fn cast (RNE); an
    # independent implementation of the same two roundings
    g = torch.Generator().manual_seed(9)
    x = torch.randn(8, 512, generator=g).to(torch.bfloat16)
    x[3] = 0
    x[5, 7] = 40.0  # one large element: the row's amax
    codes, s = oracle.quantize_activations(x.double().numpy(), "fp8")
    xf = x.float()
    amax = xf.abs().amax(dim=1)
    st = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    ref = (xf / st[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)
    assert np.array_equal(s, st.numpy())
    assert np.all(codes[3] == 0) and s[3] == 1.0
    assert codes[5, 7] == 0x7E  # the amax element maps to 448


def test_quantize_activations_mx_matches_generator_rule_and_invariants():
    g = torch.Generator().manual_seed(10)
    x = torch.randn(4, 256, generator=g).to(torch.bfloat16)
    x[1, 32:64] = 0  # an all-zero block
    codes, sb = oracle.quantize_activations(x.double().numpy(), "mxfp8")
    from routed_shared_experts_b200 import synth
    rc, rs = synth.quant_mx(x.float())
    assert np.array_equal(codes, rc.numpy()) and np.array_equal(sb, rs.numpy())
    assert sb[1, 1] == 0 and np.all(codes[1, 32:64] == 0)
    # every block's largest |code| value times 2^X stays within the block amax's e4m3 step
    vals = mo.e4m3_decode(codes).reshape(4, 8, 32) * np.ldexp(1.0, sb.astype(np.int32) - 127)[..., None]
    amax = np.abs(x.double().numpy()).reshape(4, 8, 32).max(-1)
    assert np.all(np.abs(vals).max(-1) <= amax * (1 + 2.0**-3) + 1e-30)


# ------------------------------------------------------------ router logits


def test_router_logits_small_integers_equal_the_exact_matmul():
    # integers |x|, |w| <= 8 over H = 64: every partial sum is an integer far
    # below 2^24, so any order gives the exact product; a dropped, repeated or
    # transposed term would not (T, H, E all different)
    rng = np.random.default_rng(3)
    x = rng.integers(-8, 9, (3, 64)).astype(np.float64)
    w = rng.integers(-8, 9, (64, 5)).astype(np.float64)
    got = oracle.router_logits(x, w)
    assert got.dtype == np.float32 and got.shape == (3, 5)
    assert np.array_equal(got.astype(np.float64), x @ w)
    bias = np.array([0.5, -1.0, 2.0, 0.0, 3.25])
    assert np.array_equal(oracle.router_logits(x, w, bias).astype(np.float64), x @ w + bias)


def test_router_logits_chunk_order_hand_cases():
    # H = 16, 8 chunks of 2. Row of ones against one expert column:
    # w = [2^24, 0 | 1, 1 | 0 ...]: chunk sums 2^24 and 2 add exactly
    # (2^24 + 2); one running sum over all 16 terms would stay at 2^24.
    x = np.ones((1, 16))
    w = np.zeros((16, 1))
    w[0, 0], w[2, 0], w[3, 0] = 2.0**24, 1.0, 1.0
    assert oracle.router_logits(x, w)[0, 0] == 2.0**24 + 2
    # w = [2^24, 1 | 1, 0 ...]: chunk 0 rounds 2^24 + 1 to 2^24 (ties to
    # even), then 2^24 + 1 rounds to 2^24 again: the exact sum is 2^24 + 2.
    w[:] = 0
    w[0, 0], w[1, 0], w[2, 0] = 2.0**24, 1.0, 1.0
    assert oracle.router_logits(x, w)[0, 0] == 2.0**24
    # the same three terms all inside chunk 1 round the same way
    w[:] = 0
    w[2, 0], w[3, 0] = 2.0**24, 1.0
    w[4, 0] = 1.0
    assert oracle.router_logits(x, w)[0, 0] == 2.0**24


def test_router_logits_within_the_fp32_summation_bound():
    # bf16 inputs: products exact, each of the H/8 - 1 + 7 additions on a
    # path rounds by at most 2^-24 relative to its partial sum
    g = torch.Generator().manual_seed(5)
    T, H, E = 6, 2048, 40
    x = torch.randn(T, H, generator=g).to(torch.bfloat16).double().numpy()
    w = (torch.randn(H, E, generator=g) * 0.02).to(torch.bfloat16).double().numpy()
    got = oracle.router_logits(x, w).astype(np.float64)
    exact = x @ w
    bound = (H // 8 + 8) * 2.0**-24 * (np.abs(x) @ np.abs(w))
    assert np.all(np.abs(got - exact) <= bound)
    assert np.any(got != exact)  # the rounding is really fp32


@pytest.mark.parametrize("seed", range(6))
def test_softmax_topk_brute_force_with_ties(seed):
    rng = np.random.default_rng(seed)
    E, k = 7, 3
    logits = rng.integers(-3, 3, (20, E)).astype(np.float32) * 0.5  # many exact ties
    ids, w = oracle.router_softmax_topk(logits, k, True, 1.0)
    for t in range(20):
        assert list(ids[t]) == _brute_topk(list(logits[t]), k)
        p = np.exp(logits[t].astype(np.float64))
        ref = p[ids[t]] / p[ids[t]].sum()
        np.testing.assert_allclose(w[t], ref, rtol=1e-15)


def test_softmax_topk_matches_torch_topk_on_distinct_values():
    rng = np.random.default_rng(9)
    logits = rng.normal(0, 1, (64, 32)).astype(np.float32)
    ids, w = oracle.router_softmax_topk(logits, 4, True, 1.0)
    tv, ti = torch.topk(torch.from_numpy(logits), 4, dim=1)
    assert np.array_equal(ids, ti.numpy())
    ref = torch.softmax(tv.double(), dim=1).numpy()
    np.testing.assert_allclose(w, ref, rtol=1e-14)


def test_softmax_no_renorm_is_full_softmax_and_scale_folds():
    rng = np.random.default_rng(4)
    logits = rng.normal(0, 2, (10, 16)).astype(np.float32)
    ids, w = oracle.router_softmax_topk(logits, 5, False, 1.0)
    full = torch.softmax(torch.from_numpy(logits).double(), 1).numpy()
    np.testing.assert_allclose(w, np.take_along_axis(full, ids.astype(np.int64), 1), rtol=1e-14)
    ids2, w2 = oracle.router_softmax_topk(logits, 5, True, 2.5)
    _, w1 = oracle.router_softmax_topk(logits, 5, True, 1.0)
    np.testing.assert_allclose(w2.sum(1), 2.5, rtol=1e-14)
    np.testing.assert_allclose(w2, 2.5 * w1, rtol=1e-15)


def test_sigmoid_closed_forms():
    s = mo.sigmoid_fp32(np.array([0.0, 100.0, -100.0, 2.0, -2.0], np.float32))
    assert s[0] == 0.5 and s[1] == 1.0
    assert s[2] == np.float32(1 / (1 + math.exp(100)))
    assert s[3] == np.float32(1 / (1 + math.exp(-2.0)))
    assert abs(float(s[3]) + float(s[4]) - 1.0) < 2**-23


def test_sigmoid_other_rounding_brackets_the_double_value():
    rng = np.random.default_rng(13)
    l = rng.normal(0, 3, 20000).astype(np.float32)
    v = 1.0 / (1.0 + np.exp(-l.astype(np.float64)))
    s = mo.sigmoid_fp32(l)
    o = oracle.sigmoid_fp32_other(l)
    assert np.all((np.minimum(s, o) <= v) & (v <= np.maximum(s, o)))
    # adjacent fp32 values: nothing representable strictly between them
    s32, o32 = s.astype(np.float32), o.astype(np.float32)
    assert np.all(np.nextafter(s32, o32) == o32)
    # the nearest one is the primary rounding
    assert np.all(np.abs(s - v) <= np.abs(o - v))
    # a hazard is a value (almost) on the midpoint of the two
    m = oracle.sigmoid_fp32_hazard_mask(l, margin_log2=-20)
    assert np.all(np.abs(np.abs(s - v) - np.abs(o - v))[m] <= np.abs(v[m]) * 2.0**-19)


def test_grouped_router_score_override_reproduces_default():
    rng = np.random.default_rng(14)
    l = rng.normal(0, 1, (50, 64)).astype(np.float32)
    b = rng.normal(0, 0.1, 64).astype(np.float32)
    a = oracle.router_grouped_sigmoid_topk(l, b, 6, 8, 4, True, 2.5)
    o = oracle.router_grouped_sigmoid_topk(l, b, 6, 8, 4, True, 2.5, scores=mo.sigmoid_fp32(l))
    assert np.array_equal(a[0], o[0]) and np.array_equal(a[1], o[1])


def _brute_grouped(c, s, k, n_group, topk_group, rsf):
    E = len(c)
    gsize = E // n_group
    groups = [sorted(c[g * gsize:(g + 1) * gsize], reverse=True) for g in range(n_group)]
    score = [np.float32(gr[0]) + np.float32(gr[1]) if gsize > 1 else np.float32(gr[0]) for gr in groups]
    kept = _brute_topk([float(x) for x in score], topk_group)
    allowed = [e for e in range(E) if e // gsize in kept]
    sel = sorted(allowed, key=lambda e: (-c[e], e))[:k]
    ws = np.array([float(s[e]) for e in sel])
    return sel, ws / ws.sum() * rsf


@pytest.mark.parametrize("seed", range(8))
def test_grouped_sigmoid_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    E, n_group, topk_group, k = 12, 4, 2, 3
    logits = (rng.integers(-4, 4, (16, E)) * 0.25).astype(np.float32)   # ties in c and groups
    bias = (rng.integers(-2, 2, E) * 0.125).astype(np.float32)
    ids, w = oracle.router_grouped_sigmoid_topk(logits, bias, k, n_group, topk_group, True, 2.5)
    s = mo.sigmoid_fp32(logits).astype(np.float32)
    for t in range(16):
        c = [float(np.float32(s[t, e] + bias[e])) for e in range(E)]
        sel, ref = _brute_grouped(c, s[t], k, n_group, topk_group, 2.5)
        assert list(ids[t]) == sel
        np.testing.assert_allclose(w[t], ref, rtol=1e-15)


def test_grouped_reduces_to_plain_sigmoid_topk():
    # one group, or all groups kept: plain top-k of c; zero bias: top-k of the
    # logits themselves (sigmoid is increasing; distinct logits far apart)
    rng = np.random.default_rng(21)
    logits = rng.normal(0, 1, (32, 16)).astype(np.float32)
    ref_ids, _ = oracle.router_softmax_topk(logits, 4, True, 1.0)
    for n_group, topk_group in ((1, 1), (4, 4), (16, 16)):
        ids, w = oracle.router_grouped_sigmoid_topk(logits, None, 4, n_group, topk_group, True, 1.0)
        assert np.array_equal(ids, ref_ids)
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)


def test_grouped_all_experts_selected_weights_are_normalised_scores():
    rng = np.random.default_rng(22)
    logits = rng.normal(0, 1, (5, 8)).astype(np.float32)
    ids, w = oracle.router_grouped_sigmoid_topk(logits, None, 8, 2, 2, True, 1.0)
    s = mo.sigmoid_fp32(logits)
    for t in range(5):
        assert sorted(ids[t]) == list(range(8))
        np.testing.assert_allclose(w[t], s[t, ids[t]] / s[t].sum(), rtol=1e-15)


# ---------------------------------------------------------------- sort


@pytest.mark.parametrize("T,k,E,bm", [(16, 2, 8, 16), (37, 3, 5, 4), (1, 1, 1, 8), (64, 8, 128, 16), (50, 6, 64, 128)])
def test_align_sort_matches_library_stable_sort(T, k, E, bm):
    rng = np.random.default_rng(T * 7 + E)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]) if k <= E else None
    r = oracle.align_sort(ids, E, bm)
    flat = ids.reshape(-1)
    order = np.argsort(flat, kind="stable")          # library stable sort
    real = r["sorted_ids"][r["sorted_ids"] != T * k]
    assert np.array_equal(real, order)
    assert np.array_equal(r["expert_counts"], np.bincount(flat, minlength=E))
    # invariants: every flat slot once, segments aligned to bm, single-expert blocks
    assert r["expert_counts"].sum() == T * k
    assert np.all(np.diff(r["expert_offsets"]) % bm == 0)
    assert r["num_padded"] == len(r["sorted_ids"]) <= oracle.sorted_capacity(T, k, E, bm)
    for b, e in enumerate(r["block_expert"]):
        blk = r["sorted_ids"][b * bm:(b + 1) * bm]
        assert np.all((blk == T * k) | (flat[np.minimum(blk, T * k - 1)] == e))
        assert r["expert_offsets"][e] <= b * bm < r["expert_offsets"][e + 1]
    tokens_seen = np.bincount(real // k, minlength=T)
    assert np.all(tokens_seen == k)  # each token sits in exactly k expert slots


# ---------------------------------------------------------------- gate


def test_gate_closed_form():
    K = 64
    x = np.ones((3, K))
    w = np.array([0.0, 1 / 64, -2 / 64])[:, None] * np.ones((1, K))
    for i, c in enumerate([0.0, 1.0, -2.0]):
        g = oracle.shared_gate(x[i:i + 1], w[i], True, oracle.BF16)
        assert g[0] == oracle.bf16_round(1 / (1 + math.exp(-c)))
    assert oracle.shared_gate(x[:1], w[0], True, oracle.BF16)[0] == 0.5
    g = oracle.shared_gate(x[:1], w[1] * 3, False, oracle.FP16)
    assert g[0] == 3.0


def test_gate_brute_force_dot():
    rng = np.random.default_rng(8)
    x = rng.normal(0, 1, (4, 33))
    w = rng.normal(0, 0.02, 33)
    g = oracle.shared_gate(x, w, True, oracle.FP16)
    for t in range(4):
        d = sum(x[t, i] * w[i] for i in range(33))
        assert g[t] == mo.fp16_round(1 / (1 + math.exp(-d)))


# ---------------------------------------------------------------- expert / layer


def test_silu_closed_form():
    z = np.array([0.0, 1.0, -1.0, 20.0])
    np.testing.assert_allclose(oracle.silu(z), [0.0, 1 / (1 + math.exp(-1)), -1 / (1 + math.exp(1)),
                                                20 / (1 + math.exp(-20))], rtol=1e-15)


def test_expert_forward_brute_force_loops():
    """Tiny expert written out with scalar loops: catches a transposed W13/W2,
    swapped gate/up halves, a missing SiLU or a scale in the wrong place."""
    rng = np.random.default_rng(31)
    H, I = 5, 3
    x = rng.normal(0, 1, H)
    w13 = rng.normal(0, 1, (2 * I, H))
    w2 = rng.normal(0, 1, (H, I))
    sx, s13, s2 = 0.5, 0.25, 3.0
    y = oracle.expert_forward(x, w13, w2, I, "fp8", sx, s13, s2)
    a = [sum(w13[r, c] * x[c] for c in range(H)) * sx * s13 for r in range(2 * I)]
    h = [a[i] / (1 + math.exp(-a[i])) * a[I + i] for i in range(I)]
    amax = max(abs(v) for v in h)
    s = float(np.float32(amax / 448))
    hq = [float(oracle.round_to_format(np.array([v / s]), oracle.E4M3)[0]) * s for v in h]
    ref = [sum(w2[o, i] * hq[i] for i in range(I)) * s2 for o in range(H)]
    np.testing.assert_allclose(y, ref, rtol=1e-13)


def test_expert_forward_identity_weights_closed_form():
    # W13 = [I; I] (gate = up = identity), W2 = identity: y = bf16(silu(x) * x)
    n = 8
    x = np.linspace(-3, 3, n)
    w13 = np.vstack([np.eye(n), np.eye(n)])
    y = oracle.expert_forward(x, w13, np.eye(n), n, "bf16")
    assert np.array_equal(y, oracle.bf16_round(x * x / (1 + np.exp(-x))))


def _tiny_cfg(**kw):
    cfg = dict(T=6, H=32, E=4, top_k=2, I=32, Is=32, dtype="bf16", route="softmax", n_group=1,
               topk_group=1, rsf=1.0, renormalize=True, shared_gate=True)
    cfg.update(kw)
    return cfg


def _tiny_inputs(cfg, seed=0):
    g = torch.Generator().manual_seed(seed)
    T, H, E, I, Is = (cfg[n] for n in ("T", "H", "E", "I", "Is"))
    r = lambda *s, sd=1.0: (torch.randn(*s, generator=g) * sd)  # noqa: E731
    return {"logits": r(T, E), "x": r(T, H).bfloat16(), "w_gate": r(H, sd=0.1).bfloat16(),
            "w13": r(E, 2 * I, H, sd=0.1).bfloat16(), "w2": r(E, H, I, sd=0.1).bfloat16(),
            "w13s": r(2 * Is, H, sd=0.1).bfloat16(), "w2s": r(H, Is, sd=0.1).bfloat16(),
            "correction_bias": None}


def test_layer_brute_force_tiny():
    cfg = _tiny_cfg()
    inp = _tiny_inputs(cfg)
    r = oracle.moe_layer(cfg, inp)
    x = inp["x"].double().numpy()
    lg = inp["logits"].numpy()
    for t in range(cfg["T"]):
        order = sorted(range(cfg["E"]), key=lambda e: (-lg[t, e], e))[:2]
        p = [math.exp(float(lg[t, e]) - float(lg[t, order[0]])) for e in order]
        wts = [v / sum(p) for v in p]
        d = sum(x[t, h] * float(inp["w_gate"][h]) for h in range(cfg["H"]))
        gate = float(oracle.bf16_round(np.array([1 / (1 + math.exp(-d))]))[0])

        def mlp(w13, w2, I):
            w13 = w13.double().numpy()
            w2 = w2.double().numpy()
            a = [sum(w13[i, c] * x[t, c] for c in range(cfg["H"])) for i in range(2 * I)]
            h = oracle.bf16_round(np.array([a[i] / (1 + math.exp(-a[i])) * a[I + i] for i in range(I)]))
            return np.array([sum(w2[o, i] * h[i] for i in range(I)) for o in range(cfg["H"])])
        addend = oracle.bf16_round(gate * mlp(inp["w13s"], inp["w2s"], cfg["Is"]))
        routed = sum(wts[j] * mlp(inp["w13"][order[j]], inp["w2"][order[j]], cfg["I"]) for j in range(2))
        ref = oracle.bf16_round(addend + routed)
        assert list(r["topk_ids"][t]) == order
        # brute force and oracle differ only in float64 summation order
        assert np.max(np.abs(r["out"][t] - ref)) <= 2.0**-8 * np.max(np.abs(ref)) + 1e-12


def test_layer_invariants_fold_and_addend():
    cfg = _tiny_cfg(shared_gate=False)
    inp = _tiny_inputs(cfg, seed=1)
    base = oracle.moe_layer(cfg, inp)
    scaled = oracle.moe_layer(dict(cfg, rsf=2.5), inp)
    # folding the scale into the weights == scaling the routed output
    np.testing.assert_allclose(scaled["routed"], 2.5 * base["routed"], rtol=1e-12, atol=1e-15)
    # shared expert with zero weights: the output is the routed sum alone
    zero = dict(inp, w2s=torch.zeros_like(inp["w2s"]))
    rz = oracle.moe_layer(cfg, zero)
    assert np.all(rz["addend"] == 0)
    np.testing.assert_array_equal(rz["out"], oracle.bf16_round(rz["routed"]))
    # the addend path equals a separate add of the two bf16-free parts
    np.testing.assert_array_equal(base["out"], oracle.bf16_round(base["addend"] + base["routed"]))


def test_layer_equal_logits_give_uniform_weights():
    cfg = _tiny_cfg(E=4, top_k=4, shared_gate=False)
    inp = _tiny_inputs(cfg, seed=2)
    inp["logits"] = torch.zeros(cfg["T"], 4)
    r = oracle.moe_layer(cfg, inp)
    assert np.all(r["topk_ids"] == np.arange(4))
    np.testing.assert_allclose(r["topk_weights"], 0.25, rtol=0)


def test_shared_fused_equals_the_addend_path_up_to_the_addend_rounding():
    # bf16 (h rounds per element, so cutting the shared expert into pieces does
    # not change any h value): fused out = bf16(routed + g*S), addend path out =
    # bf16(routed + bf16(g*S)); they differ only by the addend's rounding, and
    # the fused shared sum equals the addend before its rounding
    for Is in (128, 96, 320):  # Is = I, Is < I (one padded piece), Is > I (three pieces, the last padded)
        cfg = _tiny_cfg(I=128, Is=Is)
        inp = _tiny_inputs(cfg)
        a = mo.moe_layer(cfg, inp)
        f = mo.moe_layer(cfg, inp, shared_fused=True)
        assert np.array_equal(a["addend"], mo.bf16_round(f["addend"]))
        assert np.array_equal(f["out"], mo.bf16_round(f["routed"] + f["addend"]))
        # one bf16 step of the output plus the addend's rounding (a bf16 step of
        # |v| is at most |v| * 2^-7)
        ulp = (np.maximum(np.abs(a["out"]), np.abs(f["out"])) + np.abs(a["addend"])) * 2.0**-7
        assert np.all(np.abs(a["out"] - f["out"]) <= ulp + 1e-30)
        assert np.mean(a["out"] == f["out"]) > 0.5
    assert mo.shared_pieces(320, 128) == 3 and mo.shared_pieces(128, 128) == 1 and mo.shared_pieces(96, 128) == 1


def test_shared_fused_fp8_pieces_take_their_own_row_scales():
    # fp8: each piece's h row is quantised on its own I columns: with Is = 2I the
    # fused shared output equals the sum of two half-size experts, each run
    # through expert_forward on its own slice
    cfg = dict(_tiny_cfg(I=128, Is=256), dtype="fp8", shared_gate=False)
    g = np.random.default_rng(4)
    E, H, I, Is, T = cfg["E"], cfg["H"], cfg["I"], cfg["Is"], cfg["T"]
    codes = lambda *sh: g.integers(0, 0x7E, sh).astype(np.uint8) | (g.integers(0, 2, sh) * 0x80).astype(np.uint8)  # noqa: E731
    inp = {"logits": g.normal(size=(T, E)).astype(np.float32), "x": codes(T, H), "x_scale": np.full(T, 0.01),
           "w13": codes(E, 2 * I, H), "w2": codes(E, H, I), "w13_scale": np.full(E, 1e-3),
           "w2_scale": np.full(E, 1e-3), "w13s": codes(2 * Is, H), "w2s": codes(H, Is),
           "w13s_scale": np.array([2e-3]), "w2s_scale": np.array([5e-4])}
    f = mo.moe_layer(cfg, inp, shared_fused=True, tokens=[0, 3])
    x = mo.e4m3_decode(inp["x"])
    w13s, w2s = mo.e4m3_decode(inp["w13s"]), mo.e4m3_decode(inp["w2s"])
    for i, t in enumerate([0, 3]):
        want = 0.0
        for v in range(2):
            p13 = np.concatenate([w13s[v * I:(v + 1) * I], w13s[Is + v * I: Is + (v + 1) * I]])
            want = want + mo.expert_forward(x[t], p13, w2s[:, v * I:(v + 1) * I], I, "fp8", 0.01, 2e-3, 5e-4)
        assert np.allclose(f["addend"][i], want, rtol=0, atol=1e-12)


def test_layer_single_expert_is_dense_mlp():
    """E = 1, k = 1: the routed part is one dense MLP (checked with torch
    matmuls in float64 on the decoded weights)."""
    cfg = _tiny_cfg(E=1, top_k=1, shared_gate=False)
    inp = _tiny_inputs(cfg, seed=3)
    r = oracle.moe_layer(cfg, inp)
    x = inp["x"].double()
    w13 = inp["w13"][0].double()
    a = x @ w13.T
    h = torch.nn.functional.silu(a[:, :32]) * a[:, 32:]
    h = torch.from_numpy(oracle.bf16_round(h.numpy()))
    y = h @ inp["w2"][0].double().T
    np.testing.assert_allclose(r["routed"], y.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(r["topk_weights"], 1.0)


def test_fp8_layer_takes_each_experts_and_each_tokens_own_scale():
    """fp8 a8w8 (ROCm/aiter PR 6106, "Technical Details": one activation scale
    per token row, one weight scale per expert) with every expert's W13 and W2
    scale different (2^(e mod 7) * 1e-3 and 2^((e + 3) mod 5) * 2e-3) and every
    token's x scale different, against a scalar-loop brute force. Fails if the
    oracle took s[0] for every expert, swapped the W13 and W2 scales, or
    indexed the activation scale by slot or sorted row instead of by token."""
    T, H, E, k, I, Is = 7, 32, 6, 3, 32, 32
    cfg = dict(_tiny_cfg(T=T, H=H, E=E, top_k=k, I=I, Is=Is), dtype="fp8", shared_gate=False)
    g = np.random.default_rng(12)
    codes = lambda *sh: (g.integers(0, 0x70, sh).astype(np.uint8)  # noqa: E731
                         | (g.integers(0, 2, sh) * 0x80).astype(np.uint8))
    s13 = np.array([2.0 ** (e % 7) * 1e-3 for e in range(E)])
    s2 = np.array([2.0 ** ((e + 3) % 5) * 2e-3 for e in range(E)])
    sx = np.array([0.004 * (1 + 0.37 * t) for t in range(T)])
    inp = {"logits": g.normal(size=(T, E)).astype(np.float32), "x": codes(T, H), "x_scale": sx,
           "w13": codes(E, 2 * I, H), "w2": codes(E, H, I), "w13_scale": s13, "w2_scale": s2,
           "w13s": codes(2 * Is, H), "w2s": codes(H, Is), "w13s_scale": np.array([3e-3]),
           "w2s_scale": np.array([7e-4]), "correction_bias": None}
    r = oracle.moe_layer(cfg, inp)
    x = _np_table_e4m3()[inp["x"]]
    w13, w2 = _np_table_e4m3()[inp["w13"]], _np_table_e4m3()[inp["w2"]]
    w13s, w2s = _np_table_e4m3()[inp["w13s"]], _np_table_e4m3()[inp["w2s"]]

    def mlp(xt, a13, a2, inter, sxt, sa, sb):
        a = [sum(a13[i, c] * xt[c] for c in range(H)) * sxt * sa for i in range(2 * inter)]
        h = [a[i] / (1 + math.exp(-a[i])) * a[inter + i] for i in range(inter)]
        amax = max(abs(v) for v in h)
        s = float(np.float32(amax / 448)) if amax > 0 else 1.0
        hq = [_e4m3_rn(v / s) * s for v in h]
        return np.array([sum(a2[o, i] * hq[i] for i in range(inter)) * sb for o in range(H)])
    lg = inp["logits"]
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-lg[t, e], e))[:k]
        p = [math.exp(float(lg[t, e]) - float(lg[t, order[0]])) for e in order]
        wts = [v / sum(p) for v in p]
        assert list(r["topk_ids"][t]) == order
        addend = _bf16_rn(mlp(x[t], w13s, w2s, Is, sx[t], 3e-3, 7e-4))
        routed = sum(wts[j] * mlp(x[t], w13[order[j]], w2[order[j]], I, sx[t], s13[order[j]], s2[order[j]])
                     for j in range(k))
        np.testing.assert_allclose(r["addend"][t], addend, rtol=0, atol=0)
        np.testing.assert_allclose(r["routed"][t], routed, rtol=1e-12, atol=1e-15 * np.max(np.abs(routed)))
    # the same layer with one scale changed moves exactly the tokens routed to that expert
    e0 = int(r["topk_ids"][0, 0])
    bumped = dict(inp, w2_scale=np.where(np.arange(E) == e0, 2 * s2, s2))
    rb = oracle.moe_layer(cfg, bumped)
    uses = np.any(r["topk_ids"] == e0, axis=1)
    moved = np.any(rb["routed"] != r["routed"], axis=1)
    assert np.array_equal(moved, uses)


def _np_table_e4m3():
    """E4M3 values from the closed form of the format (independent of both
    oracles): sign * 2^(e-7) * (1 + m/8), subnormal 2^-6 * m/8, NaN at S.1111.111."""
    t = np.empty(256)
    for c in range(256):
        sgn = -1.0 if c & 0x80 else 1.0
        e, m = (c >> 3) & 15, c & 7
        t[c] = math.nan if (e == 15 and m == 7) else sgn * (2.0 ** -6 * m / 8 if e == 0 else 2.0 ** (e - 7) * (1 + m / 8))
    return t


def _e4m3_rn(v):
    """Nearest E4M3 value (ties to the even code), saturating at 448: scan of
    the finite non-negative values."""
    vals = _np_table_e4m3()[:0x7F]
    a = min(abs(v), 448.0)
    i = int(np.argmin(np.abs(vals - a)))
    d = abs(vals[i] - a)
    cands = [j for j in range(len(vals)) if abs(vals[j] - a) == d]
    j = [c for c in cands if c % 2 == 0][0] if len(cands) > 1 else cands[0]
    return math.copysign(vals[j], v)


def _bf16_rn(v):
    """bf16 rounding written from the format (8 significant bits, ties to
    even by Python's round) for normal-range float64 values."""
    out = []
    for x in np.ravel(np.asarray(v, np.float64)):
        if x == 0:
            out.append(x)
            continue
        _, e = math.frexp(x)  # |x| in [2^(e-1), 2^e): spacing 2^(e-1-7)
        q = 2.0 ** (e - 8)
        out.append(round(x / q) * q)
    return np.array(out).reshape(np.shape(v))
