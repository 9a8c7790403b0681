"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function ``include/moe_b200.h`` declares, and rejects invalid arguments
with the documented status before touching the device.

Invalid-argument calls pass fake device addresses; they must be refused on the
host, so these tests run only where no GPU is present (a missing check would
otherwise reach a launch)."""
import ctypes
import os
import re

import pytest
import torch

from routed_shared_experts_b200 import build, capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return capi.lib()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+|shared_expert_gate_dot)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert "moe_stage2_gemm_accumulate" in names and "shared_expert_gate_dot" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(capi.SIGNATURES)


def test_info_calls(lib):
    assert lib.moe_supports_output_addend() == 1
    assert b"sm_100a" in lib.moe_version()
    assert lib.moe_status_string(-1) == b"MOE_ERR_INVALID_ARG"
    assert lib.moe_sorted_capacity(32, 8, 128, 16) == 32 * 8 + 128 * 15  # already a multiple of 16
    assert lib.moe_sorted_capacity(5, 3, 7, 64) == 512  # 15 + 441 = 456 -> 512
    # the library's capacity is the plain bound rounded up to whole blocks
    import oracle
    for T, k, E, bm in ((5, 3, 7, 64), (32, 8, 128, 16), (1024, 6, 64, 128), (3, 2, 6, 16)):
        assert lib.moe_sorted_capacity(T, k, E, bm) == -(-oracle.sorted_capacity(T, k, E, bm) // bm) * bm
    assert lib.moe_stage2_workspace_bytes(32, 2048) == 32 * 2048 * 4 + 32 * 16 * 4
    # stage-1 workspace, 256-byte aligned parts: fp8 fp32 h + per-tile amax +
    # block counters + grid barrier; sorted token rows; MXFP8 token scale tiles
    rows = lib.moe_sorted_capacity(1024, 6, 64, 128)
    up = lambda v: (v + 255) // 256 * 256  # noqa: E731
    want = up(rows * 1408 * 4) + up(22 * rows * 4) + up(rows // 128 * 4) + 256 + up(rows * 4096)
    assert lib.moe_stage1_workspace_bytes(capi.MOE_DT_FP8_E4M3, 1024, 6, 64, 4096, 1408, 128) == want
    assert lib.moe_stage1_workspace_bytes(capi.MOE_DT_BF16, 1024, 6, 64, 4096, 1408, 128) == up(rows * 4096 * 2)
    rows16 = lib.moe_sorted_capacity(32, 8, 128, 16)
    assert lib.moe_stage1_workspace_bytes(capi.MOE_DT_BF16, 32, 8, 128, 2048, 768, 16) == up(rows16 * 2048 * 2)
    assert lib.moe_stage1_workspace_bytes(capi.MOE_DT_FP8_E4M3, 32, 8, 128, 2048, 768, 16) == \
        up(rows16 * 768 * 4) + up(12 * rows16 * 4) + up(rows16 // 16 * 4) + 256 + up(rows16 * 2048)
    rows_mx = lib.moe_sorted_capacity(4096, 8, 256, 128)
    assert lib.moe_stage1_workspace_bytes(capi.MOE_DT_MXFP8_E4M3, 4096, 8, 256, 7168, 2048, 128) == \
        up(rows_mx * 7168) + up(rows_mx // 128 * 56 * 512)
    # MXFP4 weights read the same MXFP8 token operands: same workspace
    for bm in (16, 32, 128):
        assert lib.moe_stage1_workspace_bytes(capi.MOE_DT_MXFP4_E2M1, 4096, 8, 256, 7168, 2048, bm) == \
            lib.moe_stage1_workspace_bytes(capi.MOE_DT_MXFP8_E4M3, 4096, 8, 256, 7168, 2048, bm)
    assert lib.moe_stage1_workspace_bytes(capi.MOE_DT_F32, 32, 8, 128, 2048, 768, 16) == 0
    # MXFP8 scale tiles: 512 bytes per (expert, 128-row tile, 128-column stage)
    assert lib.moe_mx_weight_scale_bytes(0, 256, 7168, 2048) == 256 * (2048 // 64) * (7168 // 128) * 512
    assert lib.moe_mx_weight_scale_bytes(1, 256, 7168, 2048) == 256 * (7168 // 128) * (2048 // 128) * 512
    assert lib.moe_mx_h_scale_bytes(4096, 8, 256, 2048, 128) == \
        lib.moe_sorted_capacity(4096, 8, 256, 128) // 128 * 16 * 512


no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="fake device addresses: CPU-only check")
P = 0x10000  # 16-byte aligned fake address, never dereferenced on the host


@no_gpu
def test_router_rejects(lib):
    f = lib.moe_router_topk
    ok = dict(l=P, b=None, T=4, E=8, k=2, mode=0, ng=1, tg=1, rn=1, rsf=1.0, ids=P, w=P)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["l"], a["b"], a["T"], a["E"], a["k"], a["mode"], a["ng"], a["tg"], a["rn"], a["rsf"], a["ids"],
                 a["w"], None)
    assert call(l=None) == -1
    assert call(T=0) == -1
    assert call(E=513) == -1
    assert call(k=9) == -1
    assert call(k=33, E=64) == -1
    assert call(mode=2) == -1
    assert call(b=P) == -1                          # bias only in grouped mode
    assert call(mode=1, ng=3) == -1                 # 3 does not divide 8
    assert call(mode=1, ng=4, tg=5) == -1
    assert call(mode=1, ng=4, tg=1, k=3) == -1      # k > topk_group * E / n_group


@no_gpu
def test_router_gemm_rejects(lib):
    f = lib.moe_router_gemm_topk

    def call(dt=capi.MOE_DT_BF16, x=P, w=P, T=4, H=256, E=8, k=2, mode=0, cb=None):
        return f(dt, x, w, None, cb, T, H, E, k, mode, 1, 1, 1, 1.0, None, P, P, None)
    assert call(dt=capi.MOE_DT_F32) == -2
    assert call(dt=capi.MOE_DT_FP8_E4M3) == -2
    assert call(x=None) == -1
    assert call(w=None) == -1
    assert call(H=252) == -4                        # H % 8
    assert call(E=12) == -4                         # E % 8 (W_r rows are bulk-copied)
    assert call(w=P + 8) == -3
    assert call(k=9) == -1
    assert call(cb=P) == -1                         # correction bias only in grouped mode


@no_gpu
def test_quantize_activations_rejects(lib):
    f = lib.moe_quantize_activations
    assert f(capi.MOE_DT_BF16, P, 4, 256, P, P, None) == -2
    assert f(capi.MOE_DT_FP8_E4M3, None, 4, 256, P, P, None) == -1
    assert f(capi.MOE_DT_FP8_E4M3, P, 0, 256, P, P, None) == -1
    assert f(capi.MOE_DT_FP8_E4M3, P, 4, 252, P, P, None) == -4     # H % 8
    assert f(capi.MOE_DT_MXFP8_E4M3, P, 4, 80, P, P, None) == -4    # H % 32
    assert f(capi.MOE_DT_FP8_E4M3, P + 8, 4, 256, P, P, None) == -3


@no_gpu
def test_append_shared_slots_rejects(lib):
    f = lib.moe_append_shared_slots
    assert f(None, P, 4, 2, 8, 1, None, 0, P, P, None) == -1
    assert f(P, P, 4, 2, 8, 0, None, 0, P, P, None) == -1          # m >= 1
    assert f(P, P, 4, 2, 512, 1, None, 0, P, P, None) == -1        # E + m <= 512
    assert f(P, P, 4, 31, 64, 2, None, 0, P, P, None) == -1        # k + m <= 32
    assert f(P, P, 4, 2, 8, 1, P, capi.MOE_DT_F32, P, P, None) == -2


@no_gpu
def test_sort_rejects(lib):
    f = lib.moe_align_sort
    assert f(None, 4, 2, 8, 16, P, P, P, P, P, None) == -1
    assert f(P, 4, 2, 8, 48, P, P, P, P, P, None) == -1       # block_m not in the set
    assert f(P, 4, 2, 600, 16, P, P, P, P, P, None) == -1     # E too large
    assert f(P, 1 << 19, 4, 8, 16, P, P, P, P, P, None) == -4  # too many slots


@no_gpu
def test_gate_rejects(lib):
    f = lib.shared_expert_gate_dot
    assert f(capi.MOE_DT_F32, P, P, 1, 8, 1, P, None) == -2
    assert f(capi.MOE_DT_BF16, None, P, 1, 8, 1, P, None) == -1
    assert f(capi.MOE_DT_BF16, P, P, 0, 8, 1, P, None) == -1


@no_gpu
def test_stage1_rejects(lib):
    f = lib.moe_stage1_gemm

    def call(dt=0, x=P, xs=None, w=P, ws=None, s=P, be=P, npd=P, T=4, k=2, H=256, I=128, E=8, bm=16, h=P, hs=None,
             w1=P):
        return f(dt, x, xs, w, ws, s, be, npd, T, k, H, I, E, bm, h, hs, w1, None)
    assert call(dt=capi.MOE_DT_F32) == -2
    assert call(x=None) == -1
    assert call(bm=24) == -1
    assert call(be=None) == -1
    assert call(s=None) == -1                       # identity routing needs top_k == 1
    assert call(dt=capi.MOE_DT_FP8_E4M3) == -1      # fp8 needs scales and h_scale
    assert call(w1=None) == -1                      # sorted token rows need the workspace
    assert call(s=None, k=1, w1=None, H=200) == -4  # identity routing needs none
    assert call(dt=capi.MOE_DT_FP8_E4M3, xs=P, ws=P, hs=P, w1=P, H=192) == -4  # fp8 K must be 128-aligned
    assert call(dt=capi.MOE_DT_MXFP8_E4M3) == -1      # MXFP8 needs its scale arrays
    assert call(dt=capi.MOE_DT_MXFP8_E4M3, xs=P, ws=P, hs=P, H=512, I=128, w1=None) == -1  # workspace
    assert call(dt=capi.MOE_DT_MXFP8_E4M3, xs=P, ws=P, hs=P, w1=P, H=512, I=192) == -3  # whole h scale tiles
    assert call(dt=capi.MOE_DT_MXFP8_E4M3, xs=P, ws=P, hs=P, w1=P, H=512, I=128, bm=256) == -1
    assert call(H=200) == -4
    assert call(I=100) == -4
    assert call(x=P + 8) == -3
    w4 = dict(dt=capi.MOE_DT_MXFP4_E2M1, xs=P, ws=P, hs=P, w1=P, H=512, I=128)
    assert call(dt=capi.MOE_DT_MXFP4_E2M1) == -1                 # scale arrays
    assert call(**dict(w4, I=192)) == -3                         # whole h scale tiles
    assert call(**dict(w4, bm=256)) == -1
    assert call(**dict(w4, H=192)) == -4                         # K stages of 128
    assert call(**dict(w4, w=P + 16)) == -3                      # e2m1 weights: 32-byte aligned


@no_gpu
def test_stage2_rejects(lib):
    f = lib.moe_stage2_gemm_accumulate

    def call(dt=0, h=P, hs=None, w2=P, w2s=None, wt=P, wdt=capi.MOE_DT_F32, s=P, be=P, npd=P, T=4, k=2, H=256,
             I=128, E=8, bm=16, add=None, ev=None, ws=P, out=P):
        return f(dt, h, hs, w2, w2s, wt, wdt, s, be, npd, T, k, H, I, E, bm, add, ev, ws, out, None)
    assert call(dt=capi.MOE_DT_FP16) == -2
    assert call(dt=capi.MOE_DT_FP8_E4M3) == -1      # fp8 needs h_scale and w2_scale
    assert call(out=None) == -1
    assert call(ws=None) == -1                      # top_k > 1 needs the workspace
    assert call(wdt=7) == -2
    assert call(H=200) == -4
    assert call(out=P + 4) == -3
    assert call(add=P + 2) == -3
    assert call(s=None) == -1
    assert call(dt=capi.MOE_DT_MXFP4_E2M1) == -1                 # h_scale and w2_scale
    assert call(dt=capi.MOE_DT_MXFP4_E2M1, hs=P, w2s=P, I=192) == -3
    assert call(dt=capi.MOE_DT_MXFP4_E2M1, hs=P, w2s=P, bm=256) == -1
    assert call(dt=capi.MOE_DT_MXFP4_E2M1, hs=P, w2s=P, w2=P + 16) == -3


def test_binding_rejects_host_tensors_before_any_call(lib):
    """The Python binding only marshals device tensors: a host tensor (whose
    address a kernel must never see) or a non-tensor is refused in Python."""
    with pytest.raises(ValueError):
        capi._ptr(torch.zeros(4))
    with pytest.raises(TypeError):
        capi._ptr([0, 1, 2])
    assert capi._ptr(None) is None
    ids = torch.zeros((4, 2), dtype=torch.int32)
    out = torch.zeros(64, dtype=torch.int32)
    with pytest.raises(ValueError):
        capi.moe_align_sort(ids, 8, 16, out, out, out, out, out)
    x = torch.zeros((4, 256), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        capi.shared_expert_gate_dot(capi.MOE_DT_BF16, x, x[0], True, torch.zeros(4, dtype=torch.bfloat16))
