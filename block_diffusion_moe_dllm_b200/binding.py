"""Thin ctypes binding of libdllm.so: the C structs of include/dllm.h and one Python function per entry point.

Argument marshalling only: tensors become device pointers and sizes, streams become cudaStream_t handles.
Every computation happens in the library's CUDA kernels. If the library is missing or fails to load, loading
raises; there is no fallback.
"""
import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libdllm.so")

OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(8)
BF16, F32 = 0, 1
FIXED, THRESHOLD = 0, 1
WEIGHTS_BF16, WEIGHTS_FP8 = 0, 1
SCORE_LOW_CONFIDENCE, SCORE_TOP_K_MARGIN, SCORE_NEG_ENTROPY = 0, 1, 2

STATUS_NAMES = {0: "DLLM_OK", 1: "DLLM_ERR_INVALID_ARG", 2: "DLLM_ERR_SHAPE", 3: "DLLM_ERR_ALIGN",
                4: "DLLM_ERR_UNSUPPORTED", 5: "DLLM_ERR_WORKSPACE", 6: "DLLM_ERR_CUDA", 7: "DLLM_ERR_TIMEOUT"}

i32, f32, vp, sz = C.c_int32, C.c_float, C.c_void_p, C.c_size_t


class GemmDesc(C.Structure):
    _fields_ = [("N", i32), ("M", i32), ("K", i32), ("ldy", i32), ("dtype", i32), ("y_f32", i32), ("residual", i32),
                ("w_fp8", i32)]


class GroupedGemmDesc(C.Structure):
    _fields_ = [("G", i32), ("rows", i32), ("K", i32), ("M", i32), ("swiglu", i32), ("extra_rows", i32),
                ("max_rows_hint", i32), ("dtype", i32), ("y_f32", i32), ("w_fp8", i32)]


class AttnDesc(C.Structure):
    _fields_ = [("B", i32), ("Lq", i32), ("Hq", i32), ("Hkv", i32), ("d", i32), ("blk_len", i32), ("q_pos0", i32),
                ("n_keys", i32), ("cap", i32), ("dtype", i32), ("scale", f32)]


class RetainDesc(C.Structure):
    _fields_ = [("B", i32), ("Hkv", i32), ("d", i32), ("P", i32), ("cap", i32), ("n_keep", i32), ("cap_thin", i32),
                ("dtype", i32), ("alpha", f32), ("n_keep_img", i32)]


class RouteDesc(C.Structure):
    _fields_ = [("Tk", i32), ("H", i32), ("E", i32), ("k", i32), ("dtype", i32)]


class ExpertDesc(C.Structure):
    _fields_ = [("Tk", i32), ("H", i32), ("E", i32), ("k", i32), ("I", i32), ("dtype", i32), ("w_fp8", i32)]


class UnmaskDesc(C.Structure):
    _fields_ = [("B", i32), ("L", i32), ("V", i32), ("max_rows", i32), ("t", i32), ("T_s", i32), ("mode", i32),
                ("tau", f32), ("k_max", i32), ("cfg", i32), ("cfg_scale", f32), ("vocab_offset", i32),
                ("dtype", i32), ("score", i32), ("cfg_image_scale", f32)]


class Layer(C.Structure):
    _fields_ = [("attn_norm", vp), ("w_qkv", vp), ("w_o", vp), ("ffn_norm", vp), ("w_router", vp),
                ("router_bias", vp), ("w_gu", vp), ("w_down", vp), ("w_gu_shared", vp), ("w_down_shared", vp),
                ("k_cache", vp), ("v_cache", vp), ("k_thin", vp), ("v_thin", vp), ("keep_pos", vp),
                ("w_gu_scale", vp), ("w_down_scale", vp), ("w_gu_shared_scale", vp), ("w_down_shared_scale", vp)]


class Model(C.Structure):
    _fields_ = [("n_layers", i32), ("H", i32), ("Hq", i32), ("Hkv", i32), ("d", i32), ("E", i32), ("k", i32),
                ("I", i32), ("V", i32), ("dtype", i32), ("eps", f32), ("rope_base", f32), ("mask_id", i32),
                ("embed", vp), ("final_norm", vp), ("w_lm", vp), ("layers", C.POINTER(Layer)),
                ("weight_format", i32), ("w_lm_scale", vp)]


class State(C.Structure):
    _fields_ = [("B", i32), ("L", i32), ("P", i32), ("cap", i32), ("cap_thin", i32), ("tokens", vp), ("mask", vp),
                ("prefix_conf", vp), ("prefix_modality", vp)]


class StepParams(C.Structure):
    _fields_ = [("t", i32), ("T_s", i32), ("mode", i32), ("tau", f32), ("k_max", i32), ("cfg", i32),
                ("cfg_scale", f32), ("vocab_offset", i32), ("vocab_len", i32), ("sprint", i32), ("n_keep", i32),
                ("retain", i32), ("commit", i32), ("sel", vp), ("nsel", vp), ("conf", vp), ("remaining", vp),
                ("score", i32), ("sprint_alpha", f32), ("n_keep_img", i32), ("cfg_image_scale", f32)]


class StepViews(C.Structure):
    _fields_ = [("logits", vp), ("row_pos", vp), ("n_rows", vp), ("x_final", vp), ("expert_counts", vp),
                ("live", vp)]


_SIGS = {
    "dllm_version": ([], C.c_char_p),
    "dllm_last_error": ([], C.c_char_p),
    "dllm_status_check": ([vp, vp], C.c_int),
    "dllm_launch_count": ([], C.c_ulonglong),
    "dllm_selftest_bounded_wait": ([vp, sz, vp], C.c_int),
    "dllm_gemm": ([C.POINTER(GemmDesc), vp, vp, vp, vp, vp, vp, sz, vp], C.c_int),
    "dllm_gemm_workspace_size": ([C.POINTER(GemmDesc)], sz),
    "dllm_grouped_gemm": ([C.POINTER(GroupedGemmDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], C.c_int),
    "dllm_grouped_gemm_workspace_size": ([C.POINTER(GroupedGemmDesc)], sz),
    "dllm_block_attn": ([C.POINTER(AttnDesc), vp, vp, vp, vp, vp, vp, sz, vp], C.c_int),
    "dllm_block_attn_workspace_size": ([C.POINTER(AttnDesc)], sz),
    "dllm_prefix_retain": ([C.POINTER(RetainDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], C.c_int),
    "dllm_prefix_retain_workspace_size": ([C.POINTER(RetainDesc)], sz),
    "dllm_moe_route": ([C.POINTER(RouteDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], C.c_int),
    "dllm_moe_route_workspace_size": ([C.POINTER(RouteDesc)], sz),
    "dllm_moe_experts": ([C.POINTER(ExpertDesc)] + [vp] * 16 + [sz, vp], C.c_int),
    "dllm_moe_experts_workspace_size": ([C.POINTER(ExpertDesc)], sz),
    "dllm_unmask": ([C.POINTER(UnmaskDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], C.c_int),
    "dllm_unmask_workspace_size": ([C.POINTER(UnmaskDesc)], sz),
    "dllm_unmask_noalloc": ([C.POINTER(UnmaskDesc), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp], C.c_int),
    "dllm_denoise_step": ([C.POINTER(Model), C.POINTER(State), C.POINTER(StepParams), vp, sz, vp], C.c_int),
    "dllm_denoise_step_workspace_size": ([C.POINTER(Model), C.POINTER(State), C.POINTER(StepParams)], sz),
    "dllm_denoise_step_views": ([C.POINTER(Model), C.POINTER(State), C.POINTER(StepParams), vp, sz,
                                 C.POINTER(StepViews)], C.c_int),
    "dllm_block_graph_create": ([C.POINTER(Model), C.POINTER(State), C.POINTER(StepParams), vp, sz, vp,
                                 C.POINTER(vp)], C.c_int),
    "dllm_block_graph_launch": ([vp, vp], C.c_int),
    "dllm_block_graph_destroy": ([vp], None),
    "dllm_block_graph_skips_finished_passes": ([vp], C.c_int),
}

EXPORTED = sorted(_SIGS)


class DllmError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


_lib = None


def load(path=LIB_PATH):
    """Load the library (once). Raises if it is missing: the package has no other implementation."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} is missing: build it with `python -m block_diffusion_moe_dllm_b200.build`")
    lib = C.CDLL(path)
    for name, (args, res) in _SIGS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def ptr(t):
    """Device (or host) address of a tensor, or None."""
    return None if t is None else t.data_ptr()


def stream_handle(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def check(code):
    if code != OK:
        raise DllmError(code, load().dllm_last_error().decode())
    return code


class Workspace:
    """Caller-owned device scratch for the library calls (a torch uint8 buffer, 256-byte aligned)."""

    def __init__(self, nbytes, device="cuda"):
        import torch
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.zeros(self.nbytes + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        self.addr = (base + 255) & ~255

    def ensure(self, nbytes):
        if nbytes > self.nbytes:
            self.__init__(nbytes, self.buf.device)
        return self


# ---------------------------------------------------------------------------------------------- call wrappers

def gemm(x, w, y, N, M, K, dtype, ldy=None, y_f32=0, residual=0, n_rows_dev=None, w_scale=None, ws=None,
         stream=None):
    """Dense projection; with w_scale given, w holds E4M3 codes (uint8) with one fp32 scale per row."""
    lib = load()
    d = GemmDesc(N, M, K, ldy or M, dtype, y_f32, residual, int(w_scale is not None))
    need = lib.dllm_gemm_workspace_size(C.byref(d))
    ws = (ws or Workspace(need, x.device)).ensure(need)
    return check(lib.dllm_gemm(C.byref(d), ptr(x), ptr(w), ptr(w_scale), ptr(y), ptr(n_rows_dev), ws.addr, ws.nbytes,
                               stream_handle(stream)))


def grouped_gemm(x, w, w_extra, counts, offsets, y, G, rows, K, M, dtype, swiglu=0, extra_rows=0, max_rows_hint=0,
                 y_f32=0, w_scale=None, w_extra_scale=None, ws=None, stream=None):
    """Grouped projection; with w_scale given, w (and w_extra) hold E4M3 codes with per-row fp32 scales."""
    lib = load()
    d = GroupedGemmDesc(G, rows, K, M, swiglu, extra_rows, max_rows_hint, dtype, y_f32, int(w_scale is not None))
    need = lib.dllm_grouped_gemm_workspace_size(C.byref(d))
    ws = (ws or Workspace(need, x.device)).ensure(need)
    return check(lib.dllm_grouped_gemm(C.byref(d), ptr(x), ptr(w), ptr(w_extra), ptr(w_scale), ptr(w_extra_scale),
                                       ptr(counts), ptr(offsets), ptr(y), ws.addr, ws.nbytes, stream_handle(stream)))


def block_attn(q, k_cache, v_cache, out, B, Lq, Hq, Hkv, d, blk_len, q_pos0, n_keys, cap, dtype, key_pos=None,
               scale=0.0, ws=None, stream=None):
    lib = load()
    desc = AttnDesc(B, Lq, Hq, Hkv, d, blk_len, q_pos0, n_keys, cap, dtype, scale)
    need = lib.dllm_block_attn_workspace_size(C.byref(desc))
    ws = (ws or Workspace(need, q.device)).ensure(need)
    return check(lib.dllm_block_attn(C.byref(desc), ptr(q), ptr(k_cache), ptr(v_cache), ptr(key_pos), ptr(out),
                                     ws.addr, ws.nbytes, stream_handle(stream)))


def prefix_retain(k_cache, v_cache, keep_pos, k_thin, v_thin, B, Hkv, d, P, cap, n_keep, cap_thin, dtype,
                  scores=None, conf=None, alpha=1.0, modality=None, n_keep_img=0, ws=None, stream=None):
    lib = load()
    desc = RetainDesc(B, Hkv, d, P, cap, n_keep, cap_thin, dtype, alpha, n_keep_img)
    need = lib.dllm_prefix_retain_workspace_size(C.byref(desc))
    ws = (ws or Workspace(need, k_cache.device)).ensure(need)
    return check(lib.dllm_prefix_retain(C.byref(desc), ptr(k_cache), ptr(v_cache), ptr(conf), ptr(modality),
                                        ptr(keep_pos), ptr(k_thin), ptr(v_thin), ptr(scores), ws.addr, ws.nbytes,
                                        stream_handle(stream)))


def moe_route(h, w_router, bias, ids, gates, counts, offsets, perm, inv, Tk, H, E, k, dtype, scores=None, ws=None,
              stream=None):
    lib = load()
    desc = RouteDesc(Tk, H, E, k, dtype)
    need = lib.dllm_moe_route_workspace_size(C.byref(desc))
    ws = (ws or Workspace(need, h.device)).ensure(need)
    return check(lib.dllm_moe_route(C.byref(desc), ptr(h), ptr(w_router), ptr(bias), ptr(ids), ptr(gates),
                                    ptr(counts), ptr(offsets), ptr(perm), ptr(inv), ptr(scores), ws.addr, ws.nbytes,
                                    stream_handle(stream)))


def moe_experts(h, w_gu, w_down, w_gu_shared, w_down_shared, counts, offsets, perm, inv, gates, x_inout, Tk, H, E,
                k, I, dtype, scales=None, ws=None, stream=None):
    """Routed + shared experts; scales = (gu, down, gu_shared, down_shared) row scales when the weights are E4M3."""
    lib = load()
    desc = ExpertDesc(Tk, H, E, k, I, dtype, int(scales is not None))
    sc = scales or (None, None, None, None)
    need = lib.dllm_moe_experts_workspace_size(C.byref(desc))
    ws = (ws or Workspace(need, h.device)).ensure(need)
    return check(lib.dllm_moe_experts(C.byref(desc), ptr(h), ptr(w_gu), ptr(w_down), ptr(w_gu_shared),
                                      ptr(w_down_shared), *[ptr(t) for t in sc], ptr(counts), ptr(offsets), ptr(perm),
                                      ptr(inv), ptr(gates), ptr(x_inout), ws.addr, ws.nbytes, stream_handle(stream)))


def unmask(logits, row_pos, n_rows_dev, tokens, mask, sel, nsel, conf, remaining, B, L, V, max_rows, t, T_s,
           dtype, mode=FIXED, tau=0.9, k_max=8, cfg=0, cfg_scale=1.0, vocab_offset=0, score=SCORE_LOW_CONFIDENCE,
           ws=None, stream=None, cfg_image_scale=1.0):
    lib = load()
    desc = UnmaskDesc(B, L, V, max_rows, t, T_s, mode, tau, k_max, cfg, cfg_scale, vocab_offset, dtype, score,
                      cfg_image_scale)
    need = lib.dllm_unmask_workspace_size(C.byref(desc))
    ws = (ws or Workspace(need, logits.device)).ensure(need)
    return check(lib.dllm_unmask(C.byref(desc), ptr(logits), ptr(row_pos), ptr(n_rows_dev), ptr(tokens), ptr(mask),
                                 ptr(sel), ptr(nsel), ptr(conf), ptr(remaining), ws.addr, ws.nbytes,
                                 stream_handle(stream)))


def status_check(ws, stream=None):
    return load().dllm_status_check(ws.addr, stream_handle(stream))


def version():
    return load().dllm_version().decode()


def launch_count():
    return int(load().dllm_launch_count())
