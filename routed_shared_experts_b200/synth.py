"""Seeded synthetic inputs of the MoE layer.

This module only draws random numbers and stores them in the layer's input
formats; it holds none of the layer's arithmetic. Both the GPU library's callers
and the CPU oracle consume the tensors it returns, byte for byte.

Draw order (one ``torch.Generator`` seeded with the config's seed, fp32 normal
draws): x, W_r, logit bias, w_gate, W13, W2, W13s, W2s, correction bias.

Input formats (the layer's inputs arrive already in their storage format):

* bf16 layers: every tensor is rounded to bf16 by ``Tensor.to(torch.bfloat16)``.
* fp8 layers: e4m3 codes (uint8) with one fp32 scale per token row of x and one
  fp32 scale per expert and matrix, scale = amax / 448, codes from torch's
  ``float8_e4m3fn`` cast of the scaled values (clamped to +-448 first).
* mxfp8 layers: e4m3 codes with one ue8m0 byte per 32 consecutive K elements of
  every row, exponent floor(log2(amax)) - 8 (clamped to [-127, 127]).
* mxfp4 layers: x as in mxfp8; the weights are drawn directly in storage
  format, uniform random bytes (two e2m1 codes each, so every one of the 16
  codes is equally likely) and ue8m0 bytes uniform in {119, 120, 121}
  (2^-8 .. 2^-6: the codes' rms of 2.9 then gives weights of rms ~0.02).
  These replace the fp32 normal draws of the weight tensors in the order above.

Router logits are the model's gate linear, which lies before the layer: they are
made here as fp32 ``x @ W_r`` (from the unrounded draws) plus a per-expert logit
bias, and handed to both sides as the same fp32 tensor. For the fused router
path the same draws are also returned in bf16: ``x_r`` (x), ``w_r`` (W_r, [H,E])
and the fp32 ``logit_bias``.
"""
from __future__ import annotations

import torch

from .configs import MoEConfig

E4M3_MAX = 448.0


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, device, std=1.0):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def _to_e4m3_codes(v: torch.Tensor) -> torch.Tensor:
    return v.clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).view(torch.uint8)


def quant_fp8_rows(v: torch.Tensor, row_dims: int):
    """Codes and fp32 scales, one scale per index of the first ``row_dims``
    dimensions (row_dims=0: one scale for the whole tensor)."""
    red = tuple(range(row_dims, v.dim()))
    amax = v.abs().amax(dim=red, keepdim=True)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    codes = _to_e4m3_codes(v / scale)
    return codes, scale.reshape(v.shape[:row_dims] if row_dims else (1,)).float()


def quant_mx(v: torch.Tensor):
    """Codes [..., K] and ue8m0 bytes [..., K/32]."""
    K = v.shape[-1]
    assert K % 32 == 0
    blk = v.reshape(v.shape[:-1] + (K // 32, 32))
    amax = blk.abs().amax(dim=-1, keepdim=True)
    _, e = torch.frexp(amax)
    X = torch.where(amax > 0, (e - 9).clamp(-127, 127), torch.full_like(e, -127))
    codes = _to_e4m3_codes(torch.ldexp(blk, (-X).float())).reshape(v.shape)
    return codes, (X.squeeze(-1) + 127).to(torch.uint8)


def _store(v: torch.Tensor, fmt: str, row_dims: int):
    if fmt == "bf16":
        return v.to(torch.bfloat16), None
    if fmt == "fp8":
        return quant_fp8_rows(v, row_dims)
    if fmt in ("mxfp8", "mxfp4"):  # mxfp4 layers: the MXFP8 activations
        return quant_mx(v)
    raise ValueError(fmt)


def draw_mxfp4(rows: int, cols: int, g, device):
    """Random MXFP4 storage: e2m1 codes [rows, cols/2] (two per byte) and
    ue8m0 bytes [rows, cols/32]."""
    codes = torch.randint(0, 256, (rows, cols // 2), generator=g, device=device, dtype=torch.uint8)
    scales = torch.randint(119, 122, (rows, cols // 32), generator=g, device=device, dtype=torch.uint8)
    return codes, scales


def make_layer_inputs(cfg: MoEConfig, device="cpu") -> dict:
    """All inputs of one layer of ``cfg`` on ``device``.

    Keys: logits, x (+ x_scale), w13 / w2 (+ _scale), w13s / w2s (+ _scale),
    w_gate (gated layers), correction_bias (or None). Weight tensors are
    generated one expert at a time so that fp32 copies of all experts never
    exist at once.
    """
    T, H, E, I, Is = cfg.T, cfg.H, cfg.E, cfg.I, cfg.Is
    g = _gen(cfg.seed, device)
    fmt = cfg.dtype
    std = cfg.weight_std

    x32 = _randn((T, H), g, device)
    w_r = _randn((H, E), g, device, std)
    if cfg.logit_bias == "normal0.5":
        lbias = _randn((E,), g, device, 0.5)
    elif cfg.logit_bias == "zipf1.2":
        rank = torch.arange(1, E + 1, device=device, dtype=torch.float32)
        lbias = 1.2 * torch.log(1.0 / rank)
    else:
        lbias = torch.zeros(E, device=device)
    logits = (x32 @ w_r + lbias[None, :]).float().contiguous()
    w_gate32 = _randn((H,), g, device, std) if cfg.shared_gate else None

    inp = {"logits": logits, "x_r": x32.to(torch.bfloat16), "w_r": w_r.to(torch.bfloat16).contiguous(),
           "logit_bias": lbias.float().contiguous()}
    # x: per-token scale (fp8) -> one scale per row
    inp["x"], inp["x_scale"] = _store(x32, fmt, 1)
    del x32
    if w_gate32 is not None:
        inp["w_gate"] = w_gate32.to(torch.bfloat16)

    def weights(rows, cols):
        if fmt == "mxfp4":
            return draw_mxfp4(rows, cols, g, device)
        return _store(_randn((rows, cols), g, device, std), fmt, 0)

    def experts(rows, cols):
        codes, scales = [], []
        for _ in range(E):
            c, s = weights(rows, cols)
            codes.append(c)
            scales.append(s)
        codes = torch.stack(codes)
        if fmt == "bf16":
            return codes, None
        return codes, torch.cat(scales) if fmt == "fp8" else torch.stack(scales)

    inp["w13"], inp["w13_scale"] = experts(2 * I, H)
    inp["w2"], inp["w2_scale"] = experts(H, I)
    inp["w13s"], inp["w13s_scale"] = weights(2 * Is, H)
    inp["w2s"], inp["w2s_scale"] = weights(H, Is)
    inp["correction_bias"] = (_randn((E,), g, device, cfg.correction_bias_std)
                              if cfg.has_correction_bias else None)
    return inp


def make_gate_inputs(K: int, dtype: str, seed: int, T: int = 1, device="cpu"):
    """Shared-gate microbenchmark inputs: x [T,K] ~ N(0,1), w [K] ~ N(0,0.02)."""
    g = _gen(seed, device)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    x = _randn((T, K), g, device).to(tdt)
    w = _randn((K,), g, device, 0.02).to(tdt)
    return x, w


def oracle_view(inp: dict) -> dict:
    """The same inputs as CPU tensors (what the oracle reads)."""
    return {k: (v.detach().cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def matrix_bytes(dtype: str, n: int) -> int:
    """Stored bytes of one weight matrix of n elements with its scales (fp8:
    one fp32 scale; MX: one byte per 32 elements)."""
    codes = {"bf16": 2 * n, "fp8": n, "mxfp8": n, "mxfp4": n // 2}[dtype]
    return codes + {"bf16": 0, "fp8": 4, "mxfp8": n // 32, "mxfp4": n // 32}[dtype]


def weight_bytes_per_expert(cfg: MoEConfig) -> int:
    """Stored bytes of one routed expert (W13 + W2 + their scales)."""
    return matrix_bytes(cfg.dtype, 2 * cfg.H * cfg.I) + matrix_bytes(cfg.dtype, cfg.H * cfg.I)


def shared_weight_bytes(cfg: MoEConfig) -> int:
    return matrix_bytes(cfg.dtype, 2 * cfg.H * cfg.Is) + matrix_bytes(cfg.dtype, cfg.H * cfg.Is)


def activation_bytes(dtype: str, rows: int, cols: int) -> int:
    """Stored bytes of a stage operand of rows x cols (x or h) with its scales
    (fp8: one fp32 per row; MX, MXFP4 layers included: one byte per 32)."""
    if dtype == "bf16":
        return 2 * rows * cols
    if dtype == "fp8":
        return rows * cols + 4 * rows
    return rows * cols + rows * cols // 32
