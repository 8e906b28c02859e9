"""The C-ABI library: it loads, exports every entry point include/dllm.h declares, and rejects bad arguments on
the host before touching the GPU (these calls launch nothing, so they run without a GPU)."""
import ctypes as C
import os
import re

import pytest

from block_diffusion_moe_dllm_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dllm.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"DLLM_API\s+[\w\s\*]+?\b(dllm_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(bd.LIB_PATH):
        from block_diffusion_moe_dllm_b200 import build
        build.build()
    return bd.load()


def test_library_exports_every_declared_symbol(lib):
    declared = _declared()
    assert len(declared) >= 17
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(bd.EXPORTED) == declared


def test_exports_nothing_else():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", bd.LIB_PATH], capture_output=True, text=True).stdout
    funcs = sorted(l.split()[-1] for l in out.splitlines() if " T " in l)
    assert funcs == _declared()


def test_version(lib):
    assert "sm_100a" in lib.dllm_version().decode()


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def test_gemm_rejects_bad_arguments(lib):
    d = bd.GemmDesc(32, 128, 64, 128, bd.BF16, 0, 0, 0)
    assert lib.dllm_gemm(C.byref(d), None, FAKE, None, FAKE, None, FAKE, 1 << 20, None) == bd.ERR_INVALID_ARG
    d.K = 0
    assert lib.dllm_gemm(C.byref(d), FAKE, FAKE, None, FAKE, None, FAKE, 1 << 20, None) == bd.ERR_SHAPE
    d.K = 64
    assert lib.dllm_gemm(C.byref(d), FAKE, FAKE, None, FAKE, None, None, 1 << 20, None) == bd.ERR_WORKSPACE
    assert lib.dllm_gemm(C.byref(d), FAKE, FAKE, None, FAKE, None, FAKE + 8, 1 << 20, None) == bd.ERR_WORKSPACE
    assert lib.dllm_gemm(C.byref(d), FAKE, FAKE, None, FAKE, None, FAKE, 16, None) == bd.ERR_WORKSPACE
    d.K = 96
    assert lib.dllm_gemm(C.byref(d), FAKE, FAKE, None, FAKE, None, FAKE, 1 << 20, None) == bd.ERR_UNSUPPORTED
    d.K = 64
    assert lib.dllm_gemm(C.byref(d), FAKE + 2, FAKE, None, FAKE, None, FAKE, 1 << 20, None) == bd.ERR_ALIGN
    assert "aligned" in lib.dllm_last_error().decode()
    # the epilogue stores 16-byte vectors: Y's base and row stride must allow them
    assert lib.dllm_gemm(C.byref(d), FAKE, FAKE, None, FAKE + 4, None, FAKE, 1 << 20, None) == bd.ERR_ALIGN
    d.ldy = 132
    assert lib.dllm_gemm(C.byref(d), FAKE, FAKE, None, FAKE, None, FAKE, 1 << 20, None) == bd.ERR_ALIGN
    assert "ldy" in lib.dllm_last_error().decode()
    d.ldy, d.w_fp8 = 128, 1             # FP8 weights without their row scales
    assert lib.dllm_gemm(C.byref(d), FAKE, FAKE, None, FAKE, None, FAKE, 1 << 20, None) == bd.ERR_INVALID_ARG
    d.residual = 1
    assert lib.dllm_gemm(C.byref(d), FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 20, None) == bd.ERR_UNSUPPORTED


def test_attention_rejects_bad_arguments(lib):
    d = bd.AttnDesc(1, 32, 16, 4, 128, 32, 1024, 1056, 1056, bd.BF16, 0.0)
    d.Hq = 15
    assert lib.dllm_block_attn(C.byref(d), FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == bd.ERR_SHAPE
    d.Hq = 16
    d.cap = 100
    assert lib.dllm_block_attn(C.byref(d), FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == bd.ERR_SHAPE
    d.cap = 1056
    d.d = 64
    assert lib.dllm_block_attn(C.byref(d), FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == bd.ERR_UNSUPPORTED


def test_route_and_experts_reject_bad_arguments(lib):
    r = bd.RouteDesc(32, 2048, 2048, 8, bd.BF16)
    args = [FAKE] * 9
    assert lib.dllm_moe_route(C.byref(r), *args, None, FAKE, 1 << 30, None) == bd.ERR_UNSUPPORTED
    r.E, r.k = 256, 300
    assert lib.dllm_moe_route(C.byref(r), *args, None, FAKE, 1 << 30, None) == bd.ERR_UNSUPPORTED
    e = bd.ExpertDesc(32, 2048, 256, 8, 512, bd.BF16, 0)
    no_scales = [None] * 4
    # one shared weight without the other
    assert lib.dllm_moe_experts(C.byref(e), FAKE, FAKE, FAKE, FAKE, None, *no_scales, FAKE, FAKE, FAKE, FAKE, FAKE,
                                FAKE, FAKE, 1 << 30, None) == bd.ERR_INVALID_ARG
    e.I = 500
    assert lib.dllm_moe_experts(C.byref(e), *([FAKE] * 5), *no_scales, *([FAKE] * 6), FAKE, 1 << 30,
                                None) == bd.ERR_UNSUPPORTED
    e.I, e.w_fp8 = 512, 1                # FP8 expert weights without their row scales
    assert lib.dllm_moe_experts(C.byref(e), *([FAKE] * 5), *no_scales, *([FAKE] * 6), FAKE, 1 << 30,
                                None) == bd.ERR_INVALID_ARG
    e.I = 192                            # FP8: K of the down projection not a multiple of 128
    assert lib.dllm_moe_experts(C.byref(e), *([FAKE] * 5), *([FAKE] * 4), *([FAKE] * 6), FAKE, 1 << 30,
                                None) == bd.ERR_UNSUPPORTED


def test_grouped_gemm_rejects_bad_arguments(lib):
    d = bd.GroupedGemmDesc(8, 64, 256, 128, 0, 0, 0, bd.BF16, 0, 0)
    args = [FAKE, FAKE, None, None, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None]
    d.K = 100
    assert lib.dllm_grouped_gemm(C.byref(d), *args) == bd.ERR_UNSUPPORTED
    d.K, d.extra_rows = 256, 8          # an extra group without its weight
    assert lib.dllm_grouped_gemm(C.byref(d), *args) == bd.ERR_INVALID_ARG
    d.extra_rows, d.swiglu, d.y_f32 = 0, 1, 1
    assert lib.dllm_grouped_gemm(C.byref(d), *args) == bd.ERR_UNSUPPORTED
    d.swiglu, d.y_f32, d.dtype = 0, 0, bd.F32
    assert lib.dllm_grouped_gemm(C.byref(d), *args) == bd.ERR_UNSUPPORTED
    d.dtype, d.w_fp8 = bd.BF16, 1        # FP8 weights without their row scales
    assert lib.dllm_grouped_gemm(C.byref(d), *args) == bd.ERR_INVALID_ARG


def test_route_workspace_covers_scores_and_permutation_segments(lib):
    """The router's workspace holds the fp32 scores, one expert histogram per permutation segment (segments of
    whole tokens, a multiple of 256 assignments, at most 128 of them) and one near-tie threshold per token."""
    import math
    lib.dllm_moe_route_workspace_size.restype = C.c_size_t
    for Tk, E, k in [(32, 256, 8), (512, 256, 8), (32768, 256, 8), (1001, 1000, 3), (5000, 96, 4), (77, 256, 6)]:
        unit = 256 // math.gcd(k, 256)
        seg_tok = max(unit, -(-(-(-Tk // 128)) // unit) * unit)
        assert (seg_tok * k) % 256 == 0
        segments = -(-Tk // seg_tok)
        assert segments <= 128
        need = Tk * E * 4 + segments * E * 4 + Tk * 4
        r = bd.RouteDesc(Tk, 2048, E, k, bd.BF16)
        assert lib.dllm_moe_route_workspace_size(C.byref(r)) >= need


def test_unmask_rejects_bad_arguments(lib):
    u = bd.UnmaskDesc(1, 64, 1024, 64, 0, 8, bd.FIXED, 0.9, 8, 0, 1.0, 0, bd.BF16)
    assert lib.dllm_unmask(C.byref(u), *([FAKE] * 10), FAKE, 1 << 30, None) == bd.ERR_SHAPE   # L > 32
    u.L, u.max_rows, u.t = 32, 32, 8
    assert lib.dllm_unmask(C.byref(u), *([FAKE] * 10), FAKE, 1 << 30, None) == bd.ERR_INVALID_ARG  # t >= T_s
    u.t, u.cfg = 0, 3                    # guidance modes are 0, 1 and 2
    assert lib.dllm_unmask(C.byref(u), *([FAKE] * 10), FAKE, 1 << 30, None) == bd.ERR_INVALID_ARG


def test_step_checks_guidance_groups(lib):
    """Editing guidance (cfg 2) needs a multiple of three rows and runs without SPRINT (the plain decode on the full
    caches); two-way guidance an even number of rows; other modes are refused. Host-side checks only."""
    layers = (bd.Layer * 1)()
    for name in ("attn_norm", "w_qkv", "w_o", "ffn_norm", "w_router", "router_bias", "w_gu", "w_down",
                 "w_gu_shared", "w_down_shared", "k_cache", "v_cache", "k_thin", "v_thin", "keep_pos"):
        setattr(layers[0], name, FAKE)
    m = bd.Model(1, 2048, 16, 4, 128, 256, 8, 512, 157184, bd.BF16, 1e-6, 1e4, 0, FAKE, FAKE, FAKE, layers)
    st = bd.State(3, 32, 1024, 1056, 544, FAKE, FAKE)
    p = bd.StepParams(0, 8, 0, 0.9, 8, 2, 4.0, 0, 0, 0, 0, 0, 0, FAKE, FAKE, FAKE, FAKE, 0, 1.0, 0, 1.5)
    size = lambda: lib.dllm_denoise_step_workspace_size(C.byref(m), C.byref(st), C.byref(p))
    assert size() > 0
    st.B = 4
    assert size() == 0 and lib.dllm_denoise_step(C.byref(m), C.byref(st), C.byref(p), FAKE, 1 << 40, None) == bd.ERR_SHAPE
    p.cfg = 1
    assert size() > 0
    st.B = 3
    assert size() == 0
    p.cfg = 3
    assert lib.dllm_denoise_step(C.byref(m), C.byref(st), C.byref(p), FAKE, 1 << 40, None) == bd.ERR_INVALID_ARG
    p.cfg, p.sprint, p.n_keep = 2, 1, 512
    assert lib.dllm_denoise_step(C.byref(m), C.byref(st), C.byref(p), FAKE, 1 << 40, None) == bd.ERR_UNSUPPORTED
    p.cfg = 0
    assert size() > 0


def test_retain_rejects_bad_arguments(lib):
    d = bd.RetainDesc(8, 4, 128, 4096, 4128, 0, 2080, bd.BF16)
    assert lib.dllm_prefix_retain(C.byref(d), FAKE, FAKE, None, None, *([FAKE] * 4), FAKE, 1 << 30, None) == bd.ERR_SHAPE
    d.n_keep, d.P, d.cap = 2048, 9000, 9100
    assert lib.dllm_prefix_retain(C.byref(d), FAKE, FAKE, None, None, *([FAKE] * 4), FAKE, 1 << 30, None) == bd.ERR_UNSUPPORTED


def test_step_rejects_bad_model(lib):
    layers = (bd.Layer * 1)()
    m = bd.Model(1, 2048, 16, 4, 128, 256, 8, 512, 157184, bd.BF16, 1e-6, 1e4, 0, FAKE, FAKE, FAKE, layers)
    st = bd.State(1, 32, 1024, 1056, 0, FAKE, FAKE)
    p = bd.StepParams(0, 8, 0, 0.9, 8, 0, 1.0, 0, 0, 0, 0, 0, 0, FAKE, FAKE, FAKE, FAKE)
    # layer 0 has NULL weights
    assert lib.dllm_denoise_step(C.byref(m), C.byref(st), C.byref(p), FAKE, 1 << 40, None) == bd.ERR_INVALID_ARG
    assert lib.dllm_denoise_step_workspace_size(C.byref(m), C.byref(st), C.byref(p)) == 0
    for name in ("attn_norm", "w_qkv", "w_o", "ffn_norm", "w_router", "router_bias", "w_gu", "w_down",
                 "w_gu_shared", "w_down_shared", "k_cache", "v_cache"):
        setattr(layers[0], name, FAKE)
    assert lib.dllm_denoise_step_workspace_size(C.byref(m), C.byref(st), C.byref(p)) > 0
    st.L = 40
    assert lib.dllm_denoise_step(C.byref(m), C.byref(st), C.byref(p), FAKE, 1 << 40, None) == bd.ERR_SHAPE
    st.L = 32
    p.t = 9
    assert lib.dllm_denoise_step(C.byref(m), C.byref(st), C.byref(p), FAKE, 1 << 40, None) == bd.ERR_INVALID_ARG
    p.t = 0
    m.d = 64
    assert lib.dllm_denoise_step(C.byref(m), C.byref(st), C.byref(p), FAKE, 1 << 40, None) == bd.ERR_UNSUPPORTED
