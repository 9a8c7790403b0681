"""CPU checks of the parity helpers that accept a different h code only at a
rounding tie (tests/gpu_helpers.py: h_flip_check). A code taken on the other
side of a tie is accepted and its difference returned; a code that differs
away from any tie fails the check."""
import numpy as np
import pytest

import oracle
from gpu_helpers import h_flip_check
from routed_shared_experts_b200 import configs


def _other_rounding(v_scaled):
    """The e4m3 neighbour on the other side of v from its nearest-even rounding."""
    q = oracle.round_to_format(v_scaled, oracle.E4M3)
    e = np.floor(np.log2(np.maximum(np.abs(v_scaled), 2.0 ** -6)))
    step = np.ldexp(1.0, (e - 3).astype(np.int32))
    return np.where(v_scaled > q, q + step, q - step)


@pytest.mark.parametrize("fmt", ["fp8", "mxfp8"])
def test_a_code_taken_at_a_tie_is_accepted_and_measured(fmt):
    cfg = configs.small(configs.FP8_A8W8 if fmt == "fp8" else configs.MXFP8_PREFILL, name="h")
    rng = np.random.default_rng(1)
    h_raw = rng.normal(0, 1, (3, 64))
    h_q = oracle.quantize_h(h_raw, fmt)
    if fmt == "fp8":
        s = oracle.fp32_round(np.max(np.abs(h_raw), axis=-1, keepdims=True) / 448.0)
    else:
        amax = np.max(np.abs(h_raw.reshape(3, 2, 32)), axis=-1, keepdims=True)
        s = np.repeat(np.ldexp(1.0, oracle.mx_block_exponent(amax).astype(np.int32)), 32, axis=-1).reshape(3, 64)
    # move element (1, 5) onto a tie of its grid (a midpoint between two codes)
    v = h_raw[1, 5] / (s[1, 0] if fmt == "fp8" else s[1, 5])
    e = np.floor(np.log2(abs(v)))
    step = 2.0 ** (e - 3)
    mid = (np.floor(abs(v) / step) + 0.5) * step * np.sign(v)
    h_raw[1, 5] = mid * (s[1, 0] if fmt == "fp8" else s[1, 5]) * (1 + 2.0 ** -30)
    h_q = oracle.quantize_h(h_raw, fmt)
    h_gpu = h_q.copy()
    sc = s[1, 0] if fmt == "fp8" else s[1, 5]
    h_gpu[1, 5] = _other_rounding(np.array([h_raw[1, 5] / sc]))[0] * sc
    if fmt == "fp8":  # codes (e4m3 values) and the GPU's row scales, one ulp off the oracle's
        gs = s[:, 0] * (1 + 2.0 ** -23)
        d = h_flip_check(cfg, (h_gpu / s, gs), h_raw, h_q)
        d0 = h_flip_check(cfg, (h_q / s, gs), h_raw, h_q)
    else:
        d = h_flip_check(cfg, h_gpu, h_raw, h_q)
        d0 = h_flip_check(cfg, h_q, h_raw, h_q)
    assert np.count_nonzero(d) == 1 and abs(d[1, 5]) == pytest.approx(step * sc)
    assert np.all(d0 == 0)


@pytest.mark.parametrize("fmt", ["fp8", "mxfp8"])
def test_a_code_differing_away_from_a_tie_is_rejected(fmt):
    cfg = configs.small(configs.FP8_A8W8 if fmt == "fp8" else configs.MXFP8_PREFILL, name="h")
    rng = np.random.default_rng(2)
    h_raw = rng.normal(0, 1, (64, 64))
    h_q = oracle.quantize_h(h_raw, fmt)
    # the element farthest from any tie, moved by one code
    i = np.unravel_index(np.argmin(np.abs(h_raw - h_q) / np.maximum(np.abs(h_raw), 1e-9)), h_raw.shape)
    h_gpu = h_q.copy()
    h_gpu[i] = h_q[i] * (1 + 2.0 ** -3)
    if fmt == "fp8":
        s = oracle.fp32_round(np.max(np.abs(h_raw), axis=-1, keepdims=True) / 448.0)
        h_gpu = (h_gpu / s, s[:, 0])
    with pytest.raises(AssertionError):
        h_flip_check(cfg, h_gpu, h_raw, h_q)
