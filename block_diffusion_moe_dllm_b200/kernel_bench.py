"""Per-kernel timing of the library's main calls at a workload's shapes (CUDA events, kernels launched alone).

    python -m block_diffusion_moe_dllm_b200.kernel_bench [--kernel lm_head|proj|experts|expert_gemms|unmask|attn|
                                                          route|all|step]
                                                         [--workload NAME] [--reps N]

Each line reports the mean time of one call, its algorithmic bytes (weights and activations it must move at
least once) and the achieved fraction of the measured HBM bandwidth. Used by bench.py for the roofline object and
as the target command of ncu captures.
"""
import argparse
import json
import os

import torch

from . import binding as bd
from . import synth
from .configs import BY_NAME, ONE_LAYER, Workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return json.load(open(p))["hbm_gbs"], "measured"
    return 6650.0, "fallback"


def tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return json.load(open(p))["bf16_tflops"], "measured"
    return 1590.0, "fallback"


def _flops(extra, flops, t):
    peak, src = tensor_peak()
    extra.update({"TFLOP/s": flops / t / 1e12, "frac_tensor": flops / t / 1e12 / peak, "tensor_peak": peak,
                  "tensor_peak_source": src})
    return extra


def timed(fn, reps, stream=None, warm=3):
    """GPU time of one call: `reps` calls captured in a CUDA graph, the replay timed with CUDA events (host-side
    launch cost excluded)."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s)
    g.replay()
    b.record(s)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / 1000.0 / max(reps, 1)


def _result(name, t, nbytes, extra=None):
    peak, src = hbm_peak()
    r = {"kernel": name, "us": t * 1e6, "bytes": nbytes, "GB/s": nbytes / t / 1e9, "frac_hbm": nbytes / t / 1e9 / peak,
         "peak_GBs": peak, "peak_source": src}
    if extra:
        r.update(extra)
    return r


def wbytes(w: Workload):
    """Bytes per element of the expert and LM-head weights (FP8 checkpoint: one, plus a 4-byte scale per row)."""
    return 1 if w.wfmt == "fp8" else 2


def bench_lm_head(w: Workload, reps, dev, stream, weights=None):
    rows = w.B * w.L   # every guidance group's rows
    if weights:
        wl, sc = weights["w_lm"], weights.get("w_lm_scale")
    else:
        wl, sc = synth.normal((w.V, w.H), w.lm_std, w.seed, "w_lm", dev, chunk_rows=16384), None
        if w.wfmt == "fp8":
            wl, sc = synth.fp8_rows(wl)
    wl = wl[w.vocab_offset: w.vocab_offset + w.vlen]
    sc = sc[w.vocab_offset: w.vocab_offset + w.vlen] if sc is not None else None
    x = synth.normal((rows, w.H), 1.0, 1, "kb_x", dev)
    y = torch.empty((rows, w.vlen), dtype=torch.bfloat16, device=dev)
    ws = bd.Workspace(1 << 16, dev)
    t = timed(lambda: bd.gemm(x, wl, y, rows, w.vlen, w.H, bd.BF16, w_scale=sc, ws=ws), reps, stream)
    nbytes = w.vlen * w.H * wbytes(w) + (w.vlen * 4 if sc is not None else 0) + rows * w.H * 2 + rows * w.vlen * 2
    return _result("gemm_tc_kernel[lm_head]", t, nbytes,
                   _flops({"rows": rows, "M": w.vlen, "K": w.H}, 2.0 * rows * w.vlen * w.H, t))


def bench_proj(w: Workload, reps, dev, stream, weights=None):
    """The dense projections of one layer at the block's row count: QKV (M = (Hq + 2 Hkv) d) and output (M = H),
    both written with a residual-free store (the step's epilogues move the same bytes)."""
    rows = w.B * w.L
    out = []
    for name, M, K in (("qkv", (w.Hq + 2 * w.Hkv) * w.d, w.H), ("o_proj", w.H, w.Hq * w.d)):
        wt = (weights["layers"][0]["w_qkv" if name == "qkv" else "w_o"] if weights else
              synth.normal((M, K), w.w_std, w.seed, f"kb_{name}", dev))
        x = synth.normal((rows, K), 1.0, 5, f"kb_{name}_x", dev)
        y = torch.empty((rows, M), dtype=torch.bfloat16, device=dev)
        ws = bd.Workspace(64 << 20, dev)
        t = timed(lambda: bd.gemm(x, wt, y, rows, M, K, bd.BF16, ws=ws), reps, stream)
        nbytes = M * K * 2 + rows * K * 2 + rows * M * 2
        out.append(_result(f"gemm_tc_kernel[{name}]", t, nbytes,
                           _flops({"rows": rows, "M": M, "K": K}, 2.0 * rows * M * K, t)))
    return out


def skewed_routing(w: Workload, rows, dev):
    """Router outputs (ids, gates, counts, offsets, perm, inv) for synth.skewed_expert_choices: the assignments
    r * k + j sorted by expert, stably (the order the library's permutation has)."""
    ids = synth.skewed_expert_choices(rows, w.E, w.k, w.seed)
    e = ids.flatten().long()
    perm = torch.sort(e, stable=True).indices.to(torch.int32)
    inv = torch.empty_like(perm)
    inv[perm.long()] = torch.arange(perm.numel(), dtype=torch.int32)
    counts = torch.bincount(e, minlength=w.E).to(torch.int32)
    offsets = torch.zeros(w.E + 1, dtype=torch.int32)
    offsets[1:] = torch.cumsum(counts, 0).to(torch.int32)
    gates = synth.uniform((rows, w.k), 0.1, 1.0, w.seed, "skewed_gates")
    gates = gates / gates.sum(1, keepdim=True)
    return tuple(t.to(dev) for t in (ids, gates, counts, offsets, perm, inv))


def bench_experts(w: Workload, reps, dev, stream, weights=None, routing="router"):
    rows = w.B * w.L
    lw = weights["layers"][0] if weights else synth.make_weights(
        Workload(**{**w.__dict__, "n_layers": 1, "V": 128}), dev)["layers"][0]
    h = synth.normal((rows, w.H), 1.0, 2, "kb_h", dev)
    ids = torch.empty((rows, w.k), dtype=torch.int32, device=dev)
    gates = torch.empty((rows, w.k), dtype=torch.float32, device=dev)
    counts = torch.empty(w.E, dtype=torch.int32, device=dev)
    offsets = torch.empty(w.E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(rows * w.k, dtype=torch.int32, device=dev)
    inv = torch.empty(rows * w.k, dtype=torch.int32, device=dev)
    ws = bd.Workspace(1 << 20, dev)
    bd.moe_route(h, lw["w_router"], lw["router_bias"], ids, gates, counts, offsets, perm, inv, rows, w.H, w.E, w.k,
                 bd.BF16, ws=ws)
    torch.cuda.synchronize()
    if routing == "skewed":
        ids, gates, counts, offsets, perm, inv = skewed_routing(w, rows, dev)
    active = int((counts > 0).sum().item())
    x = torch.zeros((rows, w.H), dtype=torch.bfloat16, device=dev)
    scales = tuple(lw[n + "_scale"] for n in ("w_gu", "w_down", "w_gu_shared", "w_down_shared")) \
        if "w_gu_scale" in lw else None
    t = timed(lambda: bd.moe_experts(h, lw["w_gu"], lw["w_down"], lw["w_gu_shared"], lw["w_down_shared"], counts,
                                     offsets, perm, inv, gates, x, rows, w.H, w.E, w.k, w.I, bd.BF16, scales=scales,
                                     ws=ws),
              reps, stream)
    nbytes = (active + 1) * 3 * w.I * w.H * wbytes(w) + 2 * rows * w.H * 2
    troute = timed(lambda: bd.moe_route(h, lw["w_router"], lw["router_bias"], ids, gates, counts, offsets, perm, inv,
                                        rows, w.H, w.E, w.k, bd.BF16, ws=ws), reps, stream)
    rbytes = w.E * w.H * 2 + rows * w.H * 2
    flops = 6.0 * w.H * w.I * (w.k + 1) * rows
    return [_result("moe_experts[gather+gemm_tc x2+combine]", t, nbytes,
                    _flops({"active_experts": active, "rows": rows}, flops, t)),
            _result("moe_route[scores+topk+permute]", troute, rbytes, {"rows": rows})]


def bench_expert_gemms(w: Workload, reps, dev, stream, weights=None, routing="router"):
    """The two grouped expert GEMMs alone (dllm_grouped_gemm, the kernels the expert call launches), at the
    workload's routed token rows (router output of random activations) plus the shared expert's rows: gate|up with
    the SwiGLU epilogue, then down with rows in the storage type (bf16), as the expert call stores them."""
    rows = w.B * w.L
    lw = weights["layers"][0] if weights else synth.make_weights(
        Workload(**{**w.__dict__, "n_layers": 1, "V": 128}), dev)["layers"][0]
    h = synth.normal((rows, w.H), 1.0, 2, "kb_h", dev)
    ids = torch.empty((rows, w.k), dtype=torch.int32, device=dev)
    gates = torch.empty((rows, w.k), dtype=torch.float32, device=dev)
    counts = torch.empty(w.E, dtype=torch.int32, device=dev)
    offsets = torch.empty(w.E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(rows * w.k, dtype=torch.int32, device=dev)
    inv = torch.empty(rows * w.k, dtype=torch.int32, device=dev)
    ws = bd.Workspace(1 << 20, dev)
    bd.moe_route(h, lw["w_router"], lw["router_bias"], ids, gates, counts, offsets, perm, inv, rows, w.H, w.E, w.k,
                 bd.BF16, ws=ws)
    torch.cuda.synchronize()
    if routing == "skewed":
        _, _, counts, offsets, _, _ = skewed_routing(w, rows, dev)
    active = int((counts > 0).sum().item())
    n = rows * w.k + rows
    hint = min(rows, max(128, 4 * ((rows * w.k + w.E - 1) // w.E)))   # the step's N-tile hint for expert GEMMs
    xp = synth.normal((n, w.H), 1.0, 6, "kb_xp", dev)
    act = torch.empty((n, w.I), dtype=torch.bfloat16, device=dev)
    y = torch.empty((n, w.H), dtype=torch.bfloat16, device=dev)
    f8 = "w_gu_scale" in lw
    sc = (lambda name: lw[name + "_scale"] if f8 else None)
    t1 = timed(lambda: bd.grouped_gemm(xp, lw["w_gu"], lw["w_gu_shared"], counts, offsets, act, w.E, n, w.H, w.I,
                                       bd.BF16, swiglu=1, extra_rows=rows, max_rows_hint=hint, w_scale=sc("w_gu"),
                                       w_extra_scale=sc("w_gu_shared"), ws=ws), reps, stream)
    t2 = timed(lambda: bd.grouped_gemm(act, lw["w_down"], lw["w_down_shared"], counts, offsets, y, w.E, n, w.I, w.H,
                                       bd.BF16, extra_rows=rows, max_rows_hint=hint, y_f32=0, w_scale=sc("w_down"),
                                       w_extra_scale=sc("w_down_shared"), ws=ws), reps, stream)
    b1 = (active + 1) * 2 * w.I * w.H * wbytes(w) + n * w.H * 2 + n * w.I * 2
    b2 = (active + 1) * w.H * w.I * wbytes(w) + n * w.I * 2 + n * w.H * 2
    f1, f2 = 2.0 * n * 2 * w.I * w.H, 2.0 * n * w.H * w.I
    return [_result("gemm_tc_kernel[experts_swiglu]", t1, b1, _flops({"active_experts": active, "rows": n}, f1, t1)),
            _result("gemm_tc_kernel[experts_down]", t2, b2, _flops({"active_experts": active, "rows": n}, f2, t2))]


def bench_unmask(w: Workload, reps, dev, stream):
    Bl = w.B // (1 + w.cfg)
    n = Bl * w.L
    logits = synth.normal(((1 + w.cfg) * n, w.vlen), 3.0, 3, "kb_logits", dev)
    row_pos = torch.arange(n, dtype=torch.int32, device=dev)
    n_dev = torch.tensor([n], dtype=torch.int32, device=dev)
    tok = torch.zeros((w.B, w.L), dtype=torch.int32, device=dev)
    msk0 = torch.ones((w.B, w.L), dtype=torch.uint8, device=dev)
    msk = msk0.clone()
    sel = torch.empty((Bl, w.L), dtype=torch.int32, device=dev)
    nsel = torch.empty(Bl, dtype=torch.int32, device=dev)
    conf = torch.empty((Bl, w.L), dtype=torch.float32, device=dev)
    rem = torch.empty(1, dtype=torch.int32, device=dev)
    ws = bd.Workspace(1 << 22, dev)

    def call():
        msk.copy_(msk0)
        bd.unmask(logits, row_pos, n_dev, tok, msk, sel, nsel, conf, rem, Bl, w.L, w.vlen, n, 0, w.T_s, bd.BF16,
                  mode=w.mode, tau=w.tau, k_max=w.k_max, cfg=w.cfg, cfg_scale=w.cfg_scale,
                  vocab_offset=w.vocab_offset, ws=ws, cfg_image_scale=w.cfg_image_scale)
    t = timed(call, reps, stream)
    nbytes = logits.numel() * 2
    return _result("unmask[reduce+select]", t, nbytes, {"rows": n, "V": w.vlen})


def bench_attn(w: Workload, reps, dev, stream):
    n_keys = (w.n_keep if w.sprint else w.P) + w.L
    cap = n_keys
    q = synth.normal((w.B, w.L, w.Hq, w.d), 1.0, 4, "kb_q", dev)
    kc = synth.normal((w.B, w.Hkv, cap, w.d), 1.0, 4, "kb_k", dev)
    vc = synth.normal((w.B, w.Hkv, cap, w.d), 1.0, 4, "kb_v", dev)
    out = torch.empty((w.B, w.L, w.Hq * w.d), dtype=torch.bfloat16, device=dev)
    ws = bd.Workspace(1 << 26, dev)
    t = timed(lambda: bd.block_attn(q, kc, vc, out, w.B, w.L, w.Hq, w.Hkv, w.d, w.L, w.P, n_keys, cap, bd.BF16,
                                    ws=ws), reps, stream)
    nbytes = 2 * w.B * w.Hkv * n_keys * w.d * 2 + 2 * w.B * w.L * w.Hq * w.d * 2
    flops = 4.0 * w.B * w.L * w.Hq * n_keys * w.d
    return _result("block_attn", t, nbytes, _flops({"keys": n_keys, "rows": w.B * w.L}, flops, t))


def bench_step(w: Workload, reps, dev, stream):
    """One whole denoising pass (dllm_denoise_step at the block's first step, every position masked) called from the
    host, timed with CUDA events around `reps` passes (the block state reset before each), after one warm-up pass.
    Also the command the pass's ncu launch list is taken with."""
    from .engine import DenoiseEngine
    wt = synth.make_weights(w, dev)
    caches = synth.make_prefix_cache(w, dev)
    tokens, mask = synth.make_block_state(w, dev)
    eng = DenoiseEngine(w, wt, caches, dev)
    eng.set_block(tokens, mask)
    eng.step(0)
    torch.cuda.synchronize()
    n0 = bd.launch_count()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    for _ in range(reps):
        eng.set_block(tokens, mask)
        a.record(stream)
        eng.step(0)
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) / 1000.0)
    t = sorted(ts)[len(ts) // 2]
    return {"kernel": "denoise_pass", "us": t * 1e6, "launches_per_pass": (bd.launch_count() - n0) // max(reps, 1),
            "rows": w.B * w.L, "layers": w.n_layers}


def bench_block(w: Workload, reps, dev, stream, trace=False):
    """One whole block (the T_s passes called from the host, then the commit pass) from the block's start state,
    after one warm-up block, timed with CUDA events. Routing and the rows of each pass are those of a real block,
    so this is the command the block's ncu launch list is taken with; `launches_before` is the number of the
    library's launches before the timed blocks (the ncu launch skip)."""
    from .engine import DenoiseEngine
    wt = synth.make_weights(w, dev)
    caches = synth.make_prefix_cache(w, dev)
    tokens, mask = synth.make_block_state(w, dev)
    eng = DenoiseEngine(w, wt, caches, dev)
    eng.set_block(tokens, mask)
    eng.decode_block()
    torch.cuda.synchronize()
    n0 = bd.launch_count()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    for _ in range(reps):
        eng.set_block(tokens, mask)     # the commit pass rewrites the same cache positions every block
        a.record(stream)
        eng.decode_block()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) / 1000.0)
    t = sorted(ts)[len(ts) // 2]
    out = {"kernel": "block", "us": t * 1e6, "launches_before": n0,
           "launches_per_block": (bd.launch_count() - n0) // max(reps, 1), "passes": w.T_s, "layers": w.n_layers}
    if trace:
        out["kernels"] = trace_block(eng, tokens, mask)
    return out


def trace_block(eng, tokens, mask):
    """Device time per kernel over one more block, from the CUDA activity trace (CUPTI through torch.profiler):
    launches, total us and share per kernel name, largest first. Kernels overlap their neighbours' tails under
    programmatic dependent launch, so the sum can exceed the block's event-timed duration slightly."""
    from torch.profiler import profile, ProfilerActivity
    eng.set_block(tokens, mask)
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        eng.decode_block()
        torch.cuda.synchronize()
    rows = {}
    for ev in prof.events():
        if ev.device_type.name != "CUDA" or not ev.name or "Memcpy" in ev.name or "Memset" in ev.name:
            continue
        r = rows.setdefault(ev.name, [0, 0.0])
        r[0] += 1
        r[1] += ev.device_time_total if hasattr(ev, "device_time_total") else ev.cuda_time_total
    total = sum(v[1] for v in rows.values()) or 1.0
    return [{"name": k, "launches": v[0], "us": round(v[1], 1), "share": round(v[1] / total, 4)}
            for k, v in sorted(rows.items(), key=lambda kv: -kv[1][1])]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", default="all")
    ap.add_argument("--workload", default=ONE_LAYER.name)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--trace", action="store_true", help="block: device time per kernel from the CUDA activity trace")
    ap.add_argument("--routing", default="router", choices=["router", "skewed"],
                    help="experts, expert_gemms: the router's choices on random activations, or the skewed choices of "
                         "a block's own routing (synth.skewed_expert_choices)")
    a = ap.parse_args()
    w = BY_NAME[a.workload]
    dev = "cuda"
    bd.load()
    stream = torch.cuda.current_stream()
    out = []
    if a.kernel in ("lm_head", "all"):
        out.append(bench_lm_head(w, a.reps, dev, stream))
    if a.kernel in ("proj", "all"):
        out.extend(bench_proj(w, a.reps, dev, stream))
    if a.kernel in ("experts", "route", "all"):
        out.extend(bench_experts(w, a.reps, dev, stream, routing=a.routing))
    if a.kernel in ("experts", "expert_gemms", "all"):
        out.extend(bench_expert_gemms(w, a.reps, dev, stream, routing=a.routing))
    if a.kernel in ("unmask", "all") and w.L <= 32:   # the prefill shape has no unmasking step
        out.append(bench_unmask(w, a.reps, dev, stream))
    if a.kernel in ("attn", "all"):
        out.append(bench_attn(w, a.reps, dev, stream))
    if a.kernel == "step":
        out.append(bench_step(w, a.reps, dev, stream))
    if a.kernel == "block":
        out.append(bench_block(w, a.reps, dev, stream, a.trace))
    for r in out:
        print(json.dumps(r), flush=True)


if __name__ == "__main__":
    main()
