"""Parity of the MXFP8 layer (e4m3 operands with one ue8m0 scale per 32 K
elements of every row, block-scaled tensor-core MMA, stage-1 output quantised
per 32 columns) with the CPU oracle.

Structured scale patterns isolate the scale layouts: with every scale byte
equal the layer is a plain e4m3 GEMM whatever the layout; scales that vary only
along rows, or only along K blocks, of one operand each exercise one index of
the scale tiles. Tolerance: 3e-2 * rms(ref) plus one bf16 step of each rounded
quantity; routing and sort bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import quantised_layer_allowance, stratified_tokens, FP8_TOL, assert_close_rms, check_routing, run_layer
from routed_shared_experts_b200 import configs, synth

pytestmark = pytest.mark.gpu

SMALL_MX = configs.small(configs.MXFP8_PREFILL, name="small_mx", T=72, H=512, E=8, top_k=2, I=256, Is=256,
                         n_group=4, topk_group=2, block_m=32, seed=31)


def _pattern(shape, kind, rng):
    """ue8m0 bytes of the given shape [..., rows, K/32]."""
    if kind == "const":
        return np.full(shape, 127, np.uint8)
    if kind == "rows":
        v = rng.integers(120, 134, shape[:-1] + (1,))
        return np.broadcast_to(v, shape).astype(np.uint8)
    if kind == "kblocks":
        v = rng.integers(120, 134, (1,) * (len(shape) - 1) + (shape[-1],))
        return np.broadcast_to(v, shape).astype(np.uint8)
    raise ValueError(kind)


def _inputs(cfg, wpat=None, xpat=None, seed=0):
    inp = synth.make_layer_inputs(cfg)
    rng = np.random.default_rng(seed)
    if wpat:
        for k in ("w13_scale", "w2_scale", "w13s_scale", "w2s_scale"):
            inp[k] = torch.from_numpy(_pattern(tuple(inp[k].shape), wpat, rng).copy())
    if xpat:
        inp["x_scale"] = torch.from_numpy(_pattern(tuple(inp["x_scale"].shape), xpat, rng).copy())
    return inp


def _check(cfg, inp, tokens=None, block_m=None):
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    layer = run_layer(cfg, dev, block_m=block_m)
    logits = inp["logits"].cpu().numpy()
    agree = check_routing(cfg, logits, None, layer.topk_ids.cpu().numpy(), layer.topk_weights.cpu().numpy())
    ids = layer.topk_ids.cpu().numpy()
    srt = oracle.align_sort(ids, cfg.E, block_m or cfg.block_m)
    n = int(layer.num_padded.item())
    assert n == srt["num_padded"]
    assert np.array_equal(layer.sorted_ids.cpu().numpy()[:n], srt["sorted_ids"])
    if isinstance(tokens, str):  # "stratified": chosen from the routing the layer took
        tokens = stratified_tokens(cfg, layer.topk_ids.cpu().numpy(), block_m)
    tokens = np.arange(cfg.T) if tokens is None else np.asarray(tokens)
    tokens = tokens[np.isin(tokens, agree)]
    # the oracle reads the generator's tensors (CPU here, or device slices one
    # expert at a time for the large layer)
    ref = oracle.moe_layer(cfg.as_dict(), inp, tokens=tokens, want_h=True)
    # h codes taken at rounding ties (checked to be ties) and their exact effect
    allow_out, allow_add, _ = quantised_layer_allowance(cfg, layer, inp, tokens, ref)
    add = layer.addend.float().cpu().numpy()[tokens]
    assert_close_rms(add, ref["addend"], FP8_TOL, "addend", allow=allow_add, exact_frac=0.95)
    out = layer.out.float().cpu().numpy()[tokens]
    return assert_close_rms(out, ref["out"], FP8_TOL, "out", rounded=[ref["out"], ref["addend"]],
                         allow=allow_out, exact_frac=0.95)


@pytest.mark.parametrize("wpat,xpat", [("const", "const"), ("rows", "const"), ("kblocks", "const"),
                                       ("const", "rows"), ("const", "kblocks"), ("rows", "kblocks")])
def test_mx_structured_scales(cuda_lib, wpat, xpat):
    _check(SMALL_MX, _inputs(SMALL_MX, wpat, xpat))


@pytest.mark.parametrize("block_m", [16, 32, 64, 128])
def test_mx_random_scales(cuda_lib, block_m):
    _check(SMALL_MX, _inputs(SMALL_MX), block_m=block_m)


@pytest.mark.parametrize("block_m", [16, 128])
def test_mx_hidden_not_multiple_of_512(cuda_lib, block_m):
    """H = 640: five 128-column K stages per tile, so the token scale tiles of
    stage 1 do not come in groups of four stages."""
    cfg = configs.small(SMALL_MX, name="small_mx_h640", H=640, seed=33)
    _check(cfg, _inputs(cfg), block_m=block_m)


def test_mx_prefill_layer(cuda_lib):
    """The full MXFP8 prefill layer on a stratified set of >= 256 tokens: one
    per active expert, the hottest expert's ragged last block, blocks spread
    over the waves of the persistent GEMMs (routing and sort: every token)."""
    cfg = configs.MXFP8_PREFILL
    inp = synth.make_layer_inputs(cfg, device="cuda")
    _check(cfg, inp, tokens="stratified")


def test_mx_pack_weight_scales_layout(cuda_lib):
    """Packed W13 / W2 scale tiles hold, at byte (m%32)*16 + (m//32)*4 + b, the
    scale of tile row m and K block b (W13 tile rows interleave 16 gate rows
    with their 16 up rows)."""
    from routed_shared_experts_b200 import capi
    E, H, I = 2, 256, 256
    rng = np.random.default_rng(5)
    w13 = rng.integers(0, 255, (E, 2 * I, H // 32), dtype=np.uint8)
    w2 = rng.integers(0, 255, (E, H, I // 32), dtype=np.uint8)
    for which, src, rows, K in ((0, w13, 2 * I, H), (1, w2, H, I)):
        dst = torch.empty(capi.mx_weight_scale_bytes(which, E, H, I), dtype=torch.uint8, device="cuda")
        capi.moe_mx_pack_weight_scales(which, torch.from_numpy(src).cuda(), dst, E, H, I)
        torch.cuda.synchronize()
        got = dst.cpu().numpy().reshape(E, -1, K // 128, 512)
        for e in range(E):
            for mt in range(got.shape[1]):
                for kg in range(K // 128):
                    for m in range(128):
                        if which == 0:
                            row = (m // 16 % 2) * I + (4 * mt + m // 32) * 16 + m % 16
                        else:
                            row = mt * 128 + m
                        for b in range(4):
                            assert got[e, mt, kg, (m % 32) * 16 + (m // 32) * 4 + b] == src[e, row, kg * 4 + b]
