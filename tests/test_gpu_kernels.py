"""Parity of the router, sort and shared-gate kernels with the CPU oracle,
called through the C ABI. Routing ids and the sort are bit-exact; top-k
weights agree to 1e-6 relative; the gate to one unit in the last place of
its output dtype."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import check_routing
from routed_shared_experts_b200 import capi, configs, synth

pytestmark = pytest.mark.gpu


def _route_gpu(logits, bias, k, mode, n_group=1, topk_group=1, renorm=True, rsf=1.0):
    T = logits.shape[0]
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    capi.moe_router_topk(logits.cuda(), None if bias is None else bias.cuda(), k, mode, n_group, topk_group,
                         renorm, rsf, ids, w)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny_bf16", "decode_bf16"])
def test_router_softmax_config(cuda_lib, name):
    cfg = configs.CONFIGS[name]
    inp = synth.make_layer_inputs(cfg)
    ids, w = _route_gpu(inp["logits"], None, cfg.top_k, capi.MOE_ROUTE_SOFTMAX, rsf=cfg.rsf)
    rid, rw = oracle.router_softmax_topk(inp["logits"].numpy(), cfg.top_k, True, cfg.rsf)
    assert np.array_equal(ids, rid)
    np.testing.assert_allclose(w, rw, rtol=1e-6)


@pytest.mark.parametrize("name", ["fp8_a8w8", "fp8_decode_T128"])
def test_router_grouped_config(cuda_lib, name):
    cfg = configs.CONFIGS[name]
    g = torch.Generator().manual_seed(cfg.seed)
    # logits and correction bias of the config's shape and distribution
    logits = torch.randn(cfg.T, cfg.E, generator=g) * 0.9
    bias = torch.randn(cfg.E, generator=g) * cfg.correction_bias_std
    ids, w = _route_gpu(logits, bias, cfg.top_k, capi.MOE_ROUTE_GROUPED_SIGMOID, cfg.n_group, cfg.topk_group,
                        True, cfg.rsf)
    check_routing(cfg, logits.numpy(), bias.numpy(), ids, w)
    np.testing.assert_allclose(w.sum(1), cfg.rsf, rtol=2e-6)


@pytest.mark.parametrize("E,k,n_group,topk_group", [(256, 8, 8, 4), (8, 2, 1, 1), (16, 16, 4, 4), (512, 32, 32, 8),
                                                    (64, 1, 32, 1)])
def test_router_grouped_shapes_with_ties(cuda_lib, E, k, n_group, topk_group):
    g = torch.Generator().manual_seed(E + k)
    # quantised logits create exact ties in c and in the group scores
    logits = (torch.randint(-6, 6, (67, E), generator=g) * 0.25).float()
    bias = (torch.randint(-2, 2, (E,), generator=g) * 0.125).float()
    ids, w = _route_gpu(logits, bias, k, capi.MOE_ROUTE_GROUPED_SIGMOID, n_group, topk_group, True, 2.5)
    rid, rw = oracle.router_grouped_sigmoid_topk(logits.numpy(), bias.numpy(), k, n_group, topk_group, True, 2.5)
    assert np.array_equal(ids, rid)
    np.testing.assert_allclose(w, rw, rtol=1e-6)


@pytest.mark.parametrize("E,k,renorm", [(8, 2, True), (128, 8, True), (128, 8, False), (512, 32, True),
                                        (33, 5, False), (1, 1, True)])
def test_router_softmax_shapes_with_ties(cuda_lib, E, k, renorm):
    g = torch.Generator().manual_seed(E * 3 + k)
    logits = (torch.randint(-4, 4, (45, E), generator=g) * 0.5).float()
    ids, w = _route_gpu(logits, None, k, capi.MOE_ROUTE_SOFTMAX, renorm=renorm, rsf=1.5)
    rid, rw = oracle.router_softmax_topk(logits.numpy(), k, renorm, 1.5)
    assert np.array_equal(ids, rid)
    np.testing.assert_allclose(w, rw, rtol=1e-6)


def test_router_fold_invariant(cuda_lib):
    """Folding rsf into the weights: rsf=2.5 weights equal 2.5 x the rsf=1
    weights (each is one fp32 rounding of the same double)."""
    g = torch.Generator().manual_seed(5)
    logits = torch.randn(100, 64, generator=g)
    _, w1 = _route_gpu(logits, None, 6, capi.MOE_ROUTE_GROUPED_SIGMOID, 8, 4, True, 1.0)
    _, w25 = _route_gpu(logits, None, 6, capi.MOE_ROUTE_GROUPED_SIGMOID, 8, 4, True, 2.5)
    np.testing.assert_allclose(w25, 2.5 * w1.astype(np.float64), rtol=2e-7)


def _sort_gpu(ids_np, E, bm):
    T, k = ids_np.shape
    cap = capi.sorted_capacity(T, k, E, bm)
    d = dict(dtype=torch.int32, device="cuda")
    ids = torch.from_numpy(ids_np.astype(np.int32)).cuda()
    sorted_ids = torch.full((cap,), -7, **d)
    block_expert = torch.full((cap // bm,), -7, **d)
    counts = torch.empty(E, **d)
    offsets = torch.empty(E + 1, **d)
    num_padded = torch.empty(1, **d)
    capi.moe_align_sort(ids, E, bm, sorted_ids, block_expert, counts, offsets, num_padded)
    torch.cuda.synchronize()
    return sorted_ids.cpu().numpy(), block_expert.cpu().numpy(), counts.cpu().numpy(), offsets.cpu().numpy(), \
        int(num_padded.item())


# T*k below and from 4096 slots on (one CTA / the 8-CTA cluster sort),
# including exactly 4095 and 4096, a ragged last cluster part, E = 512 and
# the largest batch the call accepts (T*k = 2^20)
@pytest.mark.parametrize("T,k,E,bm,skew", [(16, 2, 8, 16, 0), (32, 8, 128, 16, 0), (1024, 6, 64, 128, 0),
                                           (4096, 8, 256, 128, 1), (1, 1, 1, 16, 0), (3, 1, 512, 256, 0),
                                           (2000, 4, 16, 32, 1), (128, 6, 64, 16, 0), (5, 3, 7, 64, 0),
                                           (4095, 1, 33, 16, 0), (512, 8, 512, 64, 1), (8191, 2, 300, 256, 1),
                                           (131072, 8, 256, 128, 1)])
def test_align_sort_bit_exact(cuda_lib, T, k, E, bm, skew):
    rng = np.random.default_rng(T + E + bm)
    p = None
    if skew:
        p = 1.0 / np.arange(1, E + 1) ** 1.2
        p /= p.sum()
    if T * k > 100000:  # distinct experts per token do not matter to the sort
        ids = rng.choice(E, size=(T, k), p=p).astype(np.int32)
    else:
        ids = np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    s, be, c, o, n = _sort_gpu(ids, E, bm)
    ref = oracle.align_sort(ids, E, bm)
    assert n == ref["num_padded"]
    assert np.array_equal(s[:n], ref["sorted_ids"])
    assert np.array_equal(be[: n // bm], ref["block_expert"])
    assert np.array_equal(c, ref["expert_counts"])
    assert np.array_equal(o, ref["expert_offsets"])
    assert np.all(s[n:] == -7)  # nothing past num_padded is written


def test_align_sort_rejects_bad_ids(cuda_lib):
    ids = np.array([[0, 5], [1, 2]], np.int32)  # expert 5 of E=4 is out of range
    s, be, c, o, n = _sort_gpu(ids, 4, 16)
    assert capi.device_error() == 2
    assert c.sum() == 3


def test_align_sort_cluster_rejects_bad_ids(cuda_lib):
    rng = np.random.default_rng(5)
    ids = rng.integers(0, 64, size=(1024, 8)).astype(np.int32)
    ids[700, 3] = 64  # out of range for E = 64
    ids[1000, 0] = -1
    s, be, c, o, n = _sort_gpu(ids, 64, 128)
    assert capi.device_error() == 2
    assert c.sum() == ids.size - 2
    flat = ids.reshape(-1)
    ok = (flat >= 0) & (flat < 64)
    assert np.array_equal(c, np.bincount(flat[ok], minlength=64))
    for e in range(64):  # every valid slot in its expert's segment, ascending; the two bad ones nowhere
        assert np.array_equal(s[o[e]:o[e] + c[e]], np.nonzero(flat == e)[0])


def _ulp(v, dt):
    v = np.abs(np.asarray(v, np.float64))
    p = 8 if dt == "bf16" else 11
    emin = -126 if dt == "bf16" else -14
    _, e = np.frexp(np.maximum(v, 1e-300))
    return np.ldexp(1.0, np.maximum(e - 1, emin) - (p - 1))


@pytest.mark.parametrize("dt", ["bf16", "fp16"])
@pytest.mark.parametrize("K", [32, 1024, 2048, 4096, 65536, 131072, 1000, 7])
@pytest.mark.parametrize("sig", [True, False])
def test_shared_gate_dot(cuda_lib, dt, K, sig):
    T = 3
    x, w = synth.make_gate_inputs(K, dt, seed=K, T=T)
    out = torch.empty(T, dtype=x.dtype, device="cuda")
    capi.shared_expert_gate_dot(capi.DTYPES[dt], x.cuda(), w.cuda(), sig, out)
    torch.cuda.synchronize()
    fmt = oracle.BF16 if dt == "bf16" else oracle.FP16
    ref = oracle.shared_gate(x.double().numpy(), w.double().numpy(), sig, fmt)
    got = out.cpu().double().numpy()
    # one output ulp, plus the fp32 accumulation error bound (order of the sum
    # differs from the float64 oracle): K * 2^-24 * sum|x w|, scaled by the
    # sigmoid's slope (<= 1/4) when it is applied
    acc_err = K * 2.0**-24 * (np.abs(x.double().numpy()) @ np.abs(w.double().numpy()))
    bound = _ulp(ref, dt) + acc_err * (0.25 if sig else 1.0)
    assert np.all(np.abs(got - ref) <= bound), (got, ref, bound)


@pytest.mark.parametrize("K", [1024, 2048, 4096])
@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_shared_gate_microbench_inputs(cuda_lib, K, dt):
    x, w = synth.make_gate_inputs(K, dt, seed=configs.GATE_SEED)
    out = torch.empty(1, dtype=x.dtype, device="cuda")
    capi.shared_expert_gate_dot(capi.DTYPES[dt], x.cuda(), w.cuda(), True, out)
    torch.cuda.synchronize()
    fmt = oracle.BF16 if dt == "bf16" else oracle.FP16
    ref = oracle.shared_gate(x.double().numpy(), w.double().numpy(), True, fmt)
    assert abs(out.item() - ref[0]) <= _ulp(ref, dt)[0]
