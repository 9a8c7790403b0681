"""One MoE layer forward composed from the five C-ABI calls.

Main stream: router top-k -> align/sort -> stage 1 -> stage 2 (waits on the
addend event right before its GEMM). Side stream: shared gate -> shared stage 1
-> shared stage 2 (identity routing, top_k = 1, row weight = gate) writing the
bf16 addend -> record the addend event. This is the schedule of vllm-project/
vllm PR 65207 "Purpose", commit 2: the aux-stream shared expert overlaps
sorting and stage 1, and stage 2 accumulates its output in the epilogue.

PyTorch provides the device buffers, streams and events only; every step runs
in ``libmoe_b200.so``.
"""
from __future__ import annotations

import torch

from . import capi
from .configs import MoEConfig


def capture_forward(layer, stream=None, steps: int = 1) -> torch.cuda.CUDAGraph:
    """A CUDA graph of ``steps`` consecutive ``layer.forward(stream)`` calls.

    Replaying it enqueues the same launches on ``stream`` (both streams of the
    layer included, joined as in ``forward``). The graph reads the layer's input
    tensors and writes ``layer.out`` in place, so a caller refills the inputs
    between replays (e.g. copies of the next batch from pinned host memory on
    the same stream). The layer's workspaces stay valid across replays.
    """
    main = stream or torch.cuda.current_stream(layer.device)
    g = torch.cuda.CUDAGraph()
    main.wait_stream(torch.cuda.current_stream(layer.device))
    with torch.cuda.stream(main):
        with torch.cuda.graph(g, stream=main):
            for _ in range(steps):
                layer.forward(main)
    return g


class MoELayer:
    """Device buffers and weights of one layer; ``forward()`` enqueues a step.

    ``inp`` is a dict from ``synth.make_layer_inputs`` (tensors already on the
    device). Weights are referenced, not copied; activations (``x``,
    ``logits``) are read from the same dict at every forward, so a caller may
    refill them in place. With ``router_gemm`` the step starts from the router
    linear instead of the logits: ``moe_router_gemm_topk`` on ``x_r`` (bf16),
    ``w_r`` [H,E] and ``logit_bias``, writing the logits it used to
    ``self.logits``. With ``quantize_x`` (fp8 / MXFP8 layers) the step starts
    from the bf16 activations ``x_r``: ``moe_quantize_activations`` writes
    ``self.xq`` / ``self.xq_scale``, which both GEMM paths then read instead
    of ``x`` / ``x_scale``.
    """

    def __init__(self, cfg: MoEConfig, inp: dict, block_m: int | None = None, device=None,
                 router_gemm: bool = False, quantize_x: bool = False):
        self.cfg = cfg
        self.router_gemm = router_gemm
        if quantize_x and cfg.dtype == "bf16":
            raise ValueError("quantize_x applies to the fp8 and MXFP8 layers")
        self.quantize_x = quantize_x
        self.inp = inp
        self.device = torch.device(device or inp["x"].device)
        dev = self.device
        T, H, E, k, I, Is = cfg.T, cfg.H, cfg.E, cfg.top_k, cfg.I, cfg.Is
        self.bm = block_m or cfg.block_m
        self.dt = capi.DTYPES[cfg.dtype]
        mx = cfg.dtype in capi.MX_FORMATS
        # activation format of moe_quantize_activations (MXFP4 layers: MXFP8)
        self.qdt = capi.MOE_DT_MXFP8_E4M3 if mx else self.dt
        bm = self.bm
        cap = capi.sorted_capacity(T, k, E, bm)
        cap_s = capi.sorted_capacity(T, 1, 1, bm)  # identity rows of the shared expert
        self.cap = cap
        i32 = dict(dtype=torch.int32, device=dev)
        self.topk_ids = torch.empty((T, k), **i32)
        self.topk_weights = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.logits = torch.empty((T, E), dtype=torch.float32, device=dev) if router_gemm else None
        self.xq = self.xq_scale = None
        if quantize_x:
            self.xq = torch.empty((T, H), dtype=torch.uint8, device=dev)
            self.xq_scale = (torch.empty(T, dtype=torch.float32, device=dev) if cfg.dtype == "fp8"
                             else torch.empty((T, H // 32), dtype=torch.uint8, device=dev))
        self.sorted_ids = torch.empty(cap, **i32)
        self.block_expert = torch.empty(cap // bm, **i32)
        self.expert_counts = torch.empty(E, **i32)
        self.expert_offsets = torch.empty(E + 1, **i32)
        self.num_padded = torch.empty(1, **i32)
        # stage-1 output h in the stage-2 operand format (+ per-row scales for fp8)
        hdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.uint8
        self.h = torch.empty((cap, I), dtype=hdt, device=dev)
        self.h_s = torch.empty((cap_s, Is), dtype=hdt, device=dev)
        fp8 = cfg.dtype == "fp8"
        self.h_scale = self.h_scale_s = None
        if fp8:
            self.h_scale = torch.empty(cap, dtype=torch.float32, device=dev)
            self.h_scale_s = torch.empty(cap_s, dtype=torch.float32, device=dev)
        elif mx:
            self.h_scale = torch.zeros(capi.mx_h_scale_bytes(T, k, E, I, bm), dtype=torch.uint8, device=dev)
            self.h_scale_s = torch.zeros(capi.mx_h_scale_bytes(T, 1, 1, Is, bm), dtype=torch.uint8, device=dev)
        # MX weight scales in the kernels' tile layout (one-off preparation)
        self.wsc = {}
        for name, which, e, inter in (("w13", 0, E, I), ("w2", 1, E, I), ("w13s", 0, 1, Is), ("w2s", 1, 1, Is)):
            if mx:
                dst = torch.empty(capi.mx_weight_scale_bytes(which, e, H, inter), dtype=torch.uint8, device=dev)
                capi.moe_mx_pack_weight_scales(which, inp[name + "_scale"].contiguous(), dst, e, H, inter)
                self.wsc[name] = dst
            else:
                self.wsc[name] = inp.get(name + "_scale")
        ws1 = capi.stage1_workspace_bytes(self.dt, T, k, E, H, I, bm)
        ws1s = capi.stage1_workspace_bytes(self.dt, T, 1, 1, H, Is, bm)
        self.ws1 = torch.zeros(ws1, dtype=torch.uint8, device=dev) if ws1 else None  # zeroed once
        self.ws1_s = torch.zeros(ws1s, dtype=torch.uint8, device=dev) if ws1s else None
        gdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float16
        self.gate = torch.empty(T, dtype=gdt, device=dev) if cfg.shared_gate else None
        self.addend = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        ws = capi.stage2_workspace_bytes(T, H)
        self.acc_ws = torch.zeros(ws // 4, dtype=torch.float32, device=dev)  # zeroed once
        self.side = torch.cuda.Stream(device=dev)
        self.ev_in = torch.cuda.Event()
        self.ev_addend = torch.cuda.Event()
        self.ev_q = torch.cuda.Event()

    # -- the two halves -------------------------------------------------------

    def _x(self):
        """Stage-1 activations and their scales."""
        if self.quantize_x:
            return self.xq, self.xq_scale
        return self.inp["x"], self.inp.get("x_scale")

    def shared_expert(self, stream):
        cfg, inp = self.cfg, self.inp
        T, H, Is = cfg.T, cfg.H, cfg.Is
        if self.gate is not None:
            capi.shared_expert_gate_dot(capi.MOE_DT_BF16, inp["x"], inp["w_gate"], True, self.gate, stream)
        capi.moe_stage1_gemm(self.dt, *self._x(), inp["w13s"], self.wsc["w13s"],
                             None, None, None, T, 1, H, Is, 1, self.bm, self.h_s, self.h_scale_s, self.ws1_s, stream)
        wdt = capi.MOE_DT_BF16 if self.gate is not None else capi.MOE_DT_F32
        capi.moe_stage2_gemm_accumulate(self.dt, self.h_s, self.h_scale_s, inp["w2s"], self.wsc["w2s"],
                                        self.gate, wdt, None, None, None, T, 1, H, Is, 1, self.bm, None, None,
                                        None, self.addend, stream)

    def routed(self, stream, addend=True, probes=None, wait_x=None):
        """Main-stream half. ``probes`` = optional four events recorded on
        ``stream``: before stage 1, after stage 1, before stage 2 (after its
        wait on the addend) and after stage 2. (Each recorded event costs a few
        microseconds inside a CUDA graph; time whole steps without them.)"""
        cfg, inp = self.cfg, self.inp
        T, H, E, k, I = cfg.T, cfg.H, cfg.E, cfg.top_k, cfg.I
        mode = capi.MOE_ROUTE_SOFTMAX if cfg.route == "softmax" else capi.MOE_ROUTE_GROUPED_SIGMOID
        if self.router_gemm:
            capi.moe_router_gemm_topk(inp["x_r"], inp["w_r"], inp["logit_bias"], inp.get("correction_bias"), k,
                                      mode, cfg.n_group, cfg.topk_group, cfg.renormalize, cfg.rsf, self.logits,
                                      self.topk_ids, self.topk_weights, stream)
        else:
            capi.moe_router_topk(inp["logits"], inp.get("correction_bias"), k, mode, cfg.n_group, cfg.topk_group,
                                 cfg.renormalize, cfg.rsf, self.topk_ids, self.topk_weights, stream)
        capi.moe_align_sort(self.topk_ids, E, self.bm, self.sorted_ids, self.block_expert, self.expert_counts,
                            self.expert_offsets, self.num_padded, stream)
        if wait_x is not None:  # the quantised activations (forward with quantize_x)
            stream.wait_event(wait_x)
        if probes:
            probes[0].record(stream)
        capi.moe_stage1_gemm(self.dt, *self._x(), inp["w13"], self.wsc["w13"],
                             self.sorted_ids, self.block_expert, self.num_padded, T, k, H, I, E, self.bm, self.h,
                             self.h_scale, self.ws1, stream)
        if probes:
            probes[1].record(stream)
            if addend:  # take the addend wait before the probe: the pair times the kernel alone
                stream.wait_event(self.ev_addend)
            probes[2].record(stream)
        capi.moe_stage2_gemm_accumulate(self.dt, self.h, self.h_scale, inp["w2"], self.wsc["w2"],
                                        self.topk_weights, capi.MOE_DT_F32, self.sorted_ids, self.block_expert,
                                        self.num_padded, T, k, H, I, E, self.bm,
                                        self.addend if addend else None, self.ev_addend if addend else None,
                                        self.acc_ws, self.out, stream)
        if probes:
            probes[3].record(stream)

    def forward(self, stream=None, probes=None):
        """Enqueue one layer step on ``stream`` (default: current stream);
        returns ``self.out``. Capturable in a CUDA graph."""
        main = stream or torch.cuda.current_stream(self.device)
        self.ev_in.record(main)
        self.side.wait_event(self.ev_in)
        if self.quantize_x:
            # on the side stream, whose stage 1 needs the codes first; the main
            # stream routes and sorts meanwhile and waits only before its stage 1
            capi.moe_quantize_activations(self.qdt, self.inp["x_r"], self.xq, self.xq_scale, self.side)
            self.ev_q.record(self.side)
        self.shared_expert(self.side)
        self.ev_addend.record(self.side)
        self.routed(main, probes=probes, wait_x=self.ev_q if self.quantize_x else None)
        return self.out

    def capture(self, stream=None, steps: int = 1) -> torch.cuda.CUDAGraph:
        """``capture_forward(self, stream, steps)``: the step as a replayable graph."""
        return capture_forward(self, stream, steps)

    @property
    def launches_per_step(self) -> int:
        """Kernels this library launches per forward()."""
        cfg = self.cfg
        route = 2 + (1 if self.quantize_x else 0)  # (x quantisation,) top-k, sort
        mx = cfg.dtype in capi.MX_FORMATS
        prep_routed = 1  # sorted token copy (+ MX token scale tiles)
        prep_shared = 1 if mx else 0
        gate = 1 if self.gate is not None else 0
        return route + prep_routed + 2 + gate + prep_shared + 2


class FusedSharedMoELayer:
    """The layer with the shared expert held as m = ceil(Is / I) always-selected
    routed experts (vllm-project/vllm PR 61503 "Fused heterogeneous MoE",
    "Overview"), on one stream:

        [gate] -> top-k -> append the m shared slots (weight g_t or 1)
               -> sort over E + m experts -> stage 1 -> stage 2 (k + m slots)

    The shared weights are appended to the routed ones once, at construction:
    virtual expert E + v holds intermediate features v*I .. v*I + I - 1 of the
    shared expert (its gate rows, its up rows and its W2 columns), the last one
    zero-padded past Is, with the shared expert's weight scales. All k + m
    contributions meet in stage 2's fp32 workspace before the one bf16
    rounding: no addend, no side stream, no event. Same interface as MoELayer
    (``forward``, ``out``, ``topk_ids``, ``topk_weights``).
    """

    def __init__(self, cfg: MoEConfig, inp: dict, block_m: int | None = None, device=None):
        self.cfg = cfg
        self.inp = inp
        self.device = torch.device(device or inp["x"].device)
        dev = self.device
        T, H, E, k, I, Is = cfg.T, cfg.H, cfg.E, cfg.top_k, cfg.I, cfg.Is
        self.m = m = -(-Is // I)
        self.E2, self.k2 = E + m, k + m
        self.bm = bm = block_m or cfg.block_m
        self.dt = capi.DTYPES[cfg.dtype]
        fp8 = cfg.dtype == "fp8"
        mx = cfg.dtype in capi.MX_FORMATS
        kd = 2 if cfg.dtype == "mxfp4" else 1  # stored K elements per byte (e2m1: two)

        # combined weights [E + m, ...]: routed experts, then the shared pieces
        # (code 0 is zero in every format)
        w13s, w2s = inp["w13s"], inp["w2s"]
        p13 = torch.zeros((m, 2 * I, H // kd), dtype=w13s.dtype, device=dev)
        p2 = torch.zeros((m, H, I // kd), dtype=w2s.dtype, device=dev)
        for v in range(m):
            lo, hi = v * I, min((v + 1) * I, Is)
            p13[v, : hi - lo] = w13s[lo:hi]
            p13[v, I: I + hi - lo] = w13s[Is + lo: Is + hi]
            p2[v, :, : (hi - lo) // kd] = w2s[:, lo // kd: hi // kd]
        self.w13 = torch.cat([inp["w13"], p13]).contiguous()
        self.w2 = torch.cat([inp["w2"], p2]).contiguous()
        self.wsc = {"w13": None, "w2": None}
        if fp8:  # one fp32 scale per expert and matrix: the pieces take the shared one
            self.wsc["w13"] = torch.cat([inp["w13_scale"].reshape(-1), inp["w13s_scale"].reshape(-1).repeat(m)])
            self.wsc["w2"] = torch.cat([inp["w2_scale"].reshape(-1), inp["w2s_scale"].reshape(-1).repeat(m)])
        elif mx:  # ue8m0 rows of the pieces (127 = 1.0 on the zero padding), then the tile layout
            s13, s2 = inp["w13s_scale"], inp["w2s_scale"]
            q13 = torch.full((m, 2 * I, H // 32), 127, dtype=torch.uint8, device=dev)
            q2 = torch.full((m, H, I // 32), 127, dtype=torch.uint8, device=dev)
            for v in range(m):
                lo, hi = v * I, min((v + 1) * I, Is)
                q13[v, : hi - lo] = s13[lo:hi]
                q13[v, I: I + hi - lo] = s13[Is + lo: Is + hi]
                q2[v, :, : (hi - lo) // 32] = s2[:, lo // 32: hi // 32]
            for name, which, rows in (("w13", 0, torch.cat([inp["w13_scale"], q13])),
                                      ("w2", 1, torch.cat([inp["w2_scale"], q2]))):
                dst = torch.empty(capi.mx_weight_scale_bytes(which, self.E2, H, I), dtype=torch.uint8, device=dev)
                capi.moe_mx_pack_weight_scales(which, rows.contiguous(), dst, self.E2, H, I)
                self.wsc[name] = dst

        cap = capi.sorted_capacity(T, self.k2, self.E2, bm)
        i32 = dict(dtype=torch.int32, device=dev)
        self.topk_ids = torch.empty((T, k), **i32)
        self.topk_weights = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.ids2 = torch.empty((T, self.k2), **i32)
        self.w2slots = torch.empty((T, self.k2), dtype=torch.float32, device=dev)
        self.sorted_ids = torch.empty(cap, **i32)
        self.block_expert = torch.empty(cap // bm, **i32)
        self.expert_counts = torch.empty(self.E2, **i32)
        self.expert_offsets = torch.empty(self.E2 + 1, **i32)
        self.num_padded = torch.empty(1, **i32)
        hdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.uint8
        self.h = torch.empty((cap, I), dtype=hdt, device=dev)
        self.h_scale = None
        if fp8:
            self.h_scale = torch.empty(cap, dtype=torch.float32, device=dev)
        elif mx:
            self.h_scale = torch.zeros(capi.mx_h_scale_bytes(T, self.k2, self.E2, I, bm), dtype=torch.uint8,
                                       device=dev)
        ws1 = capi.stage1_workspace_bytes(self.dt, T, self.k2, self.E2, H, I, bm)
        self.ws1 = torch.zeros(ws1, dtype=torch.uint8, device=dev) if ws1 else None  # zeroed once
        self.gate = torch.empty(T, dtype=torch.bfloat16, device=dev) if cfg.shared_gate else None
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        self.acc_ws = torch.zeros(capi.stage2_workspace_bytes(T, H) // 4, dtype=torch.float32, device=dev)

    def forward(self, stream=None, probes=None):
        """Enqueue one layer step on ``stream``; returns ``self.out``. ``probes``:
        optional four events around stage 1 and stage 2."""
        cfg, inp = self.cfg, self.inp
        T, H, E, k, I = cfg.T, cfg.H, cfg.E, cfg.top_k, cfg.I
        s = stream or torch.cuda.current_stream(self.device)
        mode = capi.MOE_ROUTE_SOFTMAX if cfg.route == "softmax" else capi.MOE_ROUTE_GROUPED_SIGMOID
        if self.gate is not None:
            capi.shared_expert_gate_dot(capi.MOE_DT_BF16, inp["x"], inp["w_gate"], True, self.gate, s)
        capi.moe_router_topk(inp["logits"], inp.get("correction_bias"), k, mode, cfg.n_group, cfg.topk_group,
                             cfg.renormalize, cfg.rsf, self.topk_ids, self.topk_weights, s)
        capi.moe_append_shared_slots(self.topk_ids, self.topk_weights, E, self.m, self.gate, self.ids2,
                                     self.w2slots, s)
        capi.moe_align_sort(self.ids2, self.E2, self.bm, self.sorted_ids, self.block_expert, self.expert_counts,
                            self.expert_offsets, self.num_padded, s)
        if probes:
            probes[0].record(s)
        capi.moe_stage1_gemm(self.dt, inp["x"], inp.get("x_scale"), self.w13, self.wsc["w13"], self.sorted_ids,
                             self.block_expert, self.num_padded, T, self.k2, H, I, self.E2, self.bm, self.h,
                             self.h_scale, self.ws1, s)
        if probes:
            probes[1].record(s)
            probes[2].record(s)
        capi.moe_stage2_gemm_accumulate(self.dt, self.h, self.h_scale, self.w2, self.wsc["w2"], self.w2slots,
                                        capi.MOE_DT_F32, self.sorted_ids, self.block_expert, self.num_padded, T,
                                        self.k2, H, I, self.E2, self.bm, None, None, self.acc_ws, self.out, s)
        if probes:
            probes[3].record(s)
        return self.out

    def capture(self, stream=None, steps: int = 1) -> torch.cuda.CUDAGraph:
        """``capture_forward(self, stream, steps)``: the step as a replayable graph."""
        return capture_forward(self, stream, steps)

    @property
    def launches_per_step(self) -> int:
        """Kernels this library launches per forward()."""
        prep = 1  # sorted token copy (+ MX token scale tiles)
        return (1 if self.gate is not None else 0) + 3 + prep + 2
