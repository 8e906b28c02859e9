"""Decoding state of one block on the device and the denoising-step calls into the library.

``DenoiseEngine`` keeps the weights, the caches (full and SPRINT-thinned), the block state and a workspace,
fills the C structs of ``dllm_denoise_step`` with their device addresses and calls the library. It is
marshalling only: the whole pass runs in the library's kernels.
"""
import ctypes as C

import torch

from . import binding as bd
from .configs import Workload
from .synth import torch_dtype


class DenoiseEngine:
    def __init__(self, w: Workload, weights, caches, device="cuda", cap_thin=None):
        self.w = w
        self.device = device
        self.lib = bd.load()
        self.dtype = bd.BF16 if w.dtype == "bf16" else bd.F32
        self.weights = weights
        self.caches = caches
        dt = torch_dtype(w.dtype)
        n = w.n_layers
        self.cap = caches[0][0].shape[2]
        self.cap_thin = (cap_thin or (w.n_keep + w.L)) if w.sprint else 0
        self.thin = []
        self._layers = (bd.Layer * n)()
        for l in range(n):
            lw = weights["layers"][l]
            kc, vc = caches[l]
            kt = vt = kp = None
            if w.sprint:
                kt = torch.zeros((w.B, w.Hkv, self.cap_thin, w.d), dtype=dt, device=device)
                vt = torch.zeros_like(kt)
                kp = torch.zeros((w.B, self.cap_thin), dtype=torch.int32, device=device)
            self.thin.append((kt, vt, kp))
            L = self._layers[l]
            for name in ("attn_norm", "w_qkv", "w_o", "ffn_norm", "w_router", "router_bias", "w_gu", "w_down",
                         "w_gu_shared", "w_down_shared"):
                setattr(L, name, bd.ptr(lw[name]))
            L.k_cache, L.v_cache = bd.ptr(kc), bd.ptr(vc)
            L.k_thin, L.v_thin, L.keep_pos = bd.ptr(kt), bd.ptr(vt), bd.ptr(kp)
            if w.wfmt == "fp8":
                for name in ("w_gu", "w_down", "w_gu_shared", "w_down_shared"):
                    setattr(L, name + "_scale", bd.ptr(lw[name + "_scale"]))
        fp8 = w.wfmt == "fp8"
        self.model = bd.Model(n, w.H, w.Hq, w.Hkv, w.d, w.E, w.k, w.I, w.V, self.dtype, w.eps, w.rope_base,
                              w.mask_id, bd.ptr(weights["embed"]), bd.ptr(weights["final_norm"]),
                              bd.ptr(weights["w_lm"]), self._layers, bd.WEIGHTS_FP8 if fp8 else bd.WEIGHTS_BF16,
                              bd.ptr(weights["w_lm_scale"]) if fp8 else None)
        self.tokens = torch.zeros((w.B, w.L), dtype=torch.int32, device=device)
        self.mask = torch.ones((w.B, w.L), dtype=torch.uint8, device=device)
        # per-position top-1 confidences of the cache (prompt positions 1) and the prefix modality, for SPRINT's
        # mixed importance and modality counts
        self.prefix_conf = None
        self.prefix_modality = None
        if w.sprint and w.sprint_alpha < 1.0:
            self.prefix_conf = torch.ones((w.B, self.cap), dtype=torch.float32, device=device)
        if w.sprint and w.n_img_prefix:
            self.prefix_modality = torch.zeros(self.cap, dtype=torch.uint8, device=device)
            self.prefix_modality[: w.n_img_prefix] = 1
        self.state = bd.State(w.B, w.L, w.P, self.cap, self.cap_thin, bd.ptr(self.tokens), bd.ptr(self.mask),
                              bd.ptr(self.prefix_conf), bd.ptr(self.prefix_modality))
        Bl = w.B // (1 + w.cfg)
        self.sel = torch.full((Bl, w.L), -1, dtype=torch.int32, device=device)
        self.nsel = torch.zeros(Bl, dtype=torch.int32, device=device)
        self.conf = torch.zeros((Bl, w.L), dtype=torch.float32, device=device)
        self.remaining = torch.zeros(1, dtype=torch.int32, device=device)
        need = max(self._ws_size(self.params(0)), self._ws_size(self.params(0, commit=True)),
                   self._ws_size(self.params(0, retain=True)))
        if need == 0:
            raise bd.DllmError(bd.ERR_INVALID_ARG, self.lib.dllm_last_error().decode())
        self.ws = bd.Workspace(need, device)

    def _ws_size(self, p):
        return self.lib.dllm_denoise_step_workspace_size(C.byref(self.model), C.byref(self.state), C.byref(p))

    def params(self, t, commit=False, retain=None):
        w = self.w
        if retain is None:
            retain = bool(w.sprint and t == 0 and not commit)
        return bd.StepParams(t, w.T_s, w.mode, w.tau, w.k_max, w.cfg, w.cfg_scale, w.vocab_offset, w.vocab_len,
                             w.sprint, w.n_keep if w.sprint else 0, int(retain), int(commit), bd.ptr(self.sel),
                             bd.ptr(self.nsel), bd.ptr(self.conf), bd.ptr(self.remaining), w.score, w.sprint_alpha,
                             w.n_keep_img, w.cfg_image_scale)

    def set_block(self, tokens, mask):
        self.tokens.copy_(tokens)
        self.mask.copy_(mask)

    def step(self, t, stream=None, retain=None):
        p = self.params(t, retain=retain)
        return bd.check(self.lib.dllm_denoise_step(C.byref(self.model), C.byref(self.state), C.byref(p),
                                                   self.ws.addr, self.ws.nbytes, bd.stream_handle(stream)))

    def commit(self, stream=None):
        p = self.params(0, commit=True)
        return bd.check(self.lib.dllm_denoise_step(C.byref(self.model), C.byref(self.state), C.byref(p),
                                                   self.ws.addr, self.ws.nbytes, bd.stream_handle(stream)))

    def decode_block(self, stream=None):
        """All T_s denoising passes of the current block, then the commit pass."""
        for t in range(self.w.T_s):
            self.step(t, stream)
        self.commit(stream)

    def capture_block(self, tokens0=None, mask0=None):
        """A CUDA graph of one block: optional reset of the block state from device tensors, the T_s passes and the
        commit pass, captured once (kernel launches and their arguments are fixed; the block's data is not)."""
        for _ in range(2):                                  # warm the library's one-time set-up outside capture
            if tokens0 is not None:
                self.set_block(tokens0, mask0)
            self.decode_block()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            if tokens0 is not None:
                self.tokens.copy_(tokens0)
                self.mask.copy_(mask0)
            self.decode_block(torch.cuda.current_stream())
        return g

    def block_graph(self, capture_stream=None):
        """The library's block graph (dllm_block_graph_create): the T_s passes, each run only while the block has
        masked positions, and the commit pass, captured once on a side stream. Warm the library's one-time set-up
        (one decode_block) before the first call."""
        return BlockGraph(self, capture_stream or torch.cuda.Stream(self.device))

    def views(self, t=0):
        p = self.params(t)
        v = bd.StepViews()
        bd.check(self.lib.dllm_denoise_step_views(C.byref(self.model), C.byref(self.state), C.byref(p),
                                                  self.ws.addr, self.ws.nbytes, C.byref(v)))
        return v

    def logits(self, n_rows):
        """The last pass's logits [rows, vlen] as a tensor view of the workspace."""
        w = self.w
        v = self.views()
        halves = 1 + w.cfg
        numel = halves * n_rows * w.vlen
        dt = torch_dtype(w.dtype)
        return _device_view(v.logits, numel, dt, self.ws.buf).reshape(halves * n_rows, w.vlen)

    def expert_counts(self, v=None):
        """Per layer, the assignments routed to each expert by the last pass that ran the layer: [n_layers, E + 1]
        int32 view of the workspace (entry E unused)."""
        w = self.w
        v = v or self.views()
        return _device_view(v.expert_counts, w.n_layers * (w.E + 1), torch.int32, self.ws.buf).reshape(
            w.n_layers, w.E + 1)

    def x_final(self):
        w = self.w
        v = self.views()
        return _device_view(v.x_final, w.Tk * w.H, torch_dtype(w.dtype), self.ws.buf).reshape(w.Tk, w.H)


class BlockGraph:
    """Owner of a dllm_block_graph handle (destroyed with the object)."""

    def __init__(self, eng, capture_stream):
        self.lib = eng.lib
        self.eng = eng                     # keeps the tensors the graph's kernels address alive
        self.handle = C.c_void_p()
        p = eng.params(0)
        bd.check(self.lib.dllm_block_graph_create(C.byref(eng.model), C.byref(eng.state), C.byref(p), eng.ws.addr,
                                                  eng.ws.nbytes, bd.stream_handle(capture_stream),
                                                  C.byref(self.handle)))
        # why the passes are unconditional, when they are (the library leaves it in the last-error text)
        self.note = "" if self.conditional else self.lib.dllm_last_error().decode()

    def launch(self, stream=None):
        return bd.check(self.lib.dllm_block_graph_launch(self.handle, bd.stream_handle(stream)))

    @property
    def conditional(self):
        """True when the passes sit in conditional nodes (passes after an early finish are not launched)."""
        return bool(self.lib.dllm_block_graph_skips_finished_passes(self.handle))

    def __del__(self):
        if getattr(self, "handle", None) and self.handle.value:
            self.lib.dllm_block_graph_destroy(self.handle)
            self.handle = C.c_void_p()


def _device_view(addr, numel, dtype, owner):
    """A tensor over ``numel`` elements at device address ``addr`` inside ``owner`` (a uint8 buffer)."""
    off = addr - owner.data_ptr()
    es = torch.empty((), dtype=dtype).element_size()
    return owner[off: off + numel * es].view(dtype)
