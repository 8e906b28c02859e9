"""Benchmark of the block-diffusion denoising step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

Default workload: understanding (20 layers, batch 16, hidden 2048, 16 q heads x 128, 4 kv heads, 256 experts top-8
+ shared, inter 512, vocab 157184, prefix 2688, block 32, 32 steps per block, threshold acceptance tau 0.9 with at
most 8 tokens per step), the largest configuration that fits one GPU.

One bench step decodes one block: the block state is reset from a device copy, then the library's block graph
(dllm_block_graph_create) runs its T_s denoising passes (embedding, attention over the cached prefix, MoE FFN, LM
head over the still-masked rows, confidence + unmasking) and the commit pass that writes the block's clean K/V
into the cache. Threshold acceptance can finish a block before its last step; each pass sits in a conditional
node that runs it only while masked positions are left. Metric: denoise-step tokens/s = B * L tokens for every pass
that ran, per second. Also reported: committed tokens/s (the block's B' * L tokens per block
time), the live passes per block, the experts each layer routed to, and the step's algorithmic bytes against HBM.

Timing: K steps between CUDA events after W warm-up steps, repeated until the timed units cover at least 2 s; the
median unit is reported. Weights streamed per pass (tens of GB) exceed the 126 MB L2, so no flush is needed.

With N > 1 (torchrun), every rank decodes its own replica (independent requests, no collective on the data
path): value = tokens of all ranks / max over ranks of the timed region.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_diffusion_moe_dllm_b200.configs import BY_NAME, UNDERSTANDING, scaled  # noqa: E402

METRIC = "denoise-step tokens/s (bf16, 1 B200)"
SPEC_HBM_GBS = 8000.0       # the ~8 TB/s HBM3e figure the targets are quoted against (context beside the measured)
MIN_TIMED_S = 2.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=UNDERSTANDING.name)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8-checkpoint leg")
    return ap.parse_args()


def dist_env():
    from block_diffusion_moe_dllm_b200 import replicas
    return replicas.env()


def bench_config(w, world):
    """The workload description both arms print (identical keys and values)."""
    return {"workload": w.name, "B": w.B, "L": w.L, "T_s": w.T_s, "P": w.P, "H": w.H, "Hq": w.Hq, "Hkv": w.Hkv,
            "d": w.d, "E": w.E, "k": w.k, "I": w.I, "V": w.V, "vocab_scored": w.vlen, "layers": w.n_layers,
            "weights": "fp8 e4m3 experts + lm head, per-row fp32 scales" if w.wfmt == "fp8" else "bf16",
            "mode": "threshold" if w.mode else "fixed", "tau": w.tau if w.mode else None,
            "k_max": w.k_max if w.mode else None, "cfg": w.cfg_scale if w.cfg else None,
            **({"cfg_image": w.cfg_image_scale} if w.cfg == 2 else {}),
            "sprint_keep": w.keep_ratio if w.sprint else None,
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2 (weights streamed per pass)"}


# ---------------------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix=f"dllm_clocks_{gpu_index}_", suffix=".csv")
        os.close(fd)

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for name, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "samples_under_load": len(loaded)}


# ---------------------------------------------------------------------------------------------- CPU oracle
class OracleSample:
    """The fp64 oracle timed on a bounded sample of the workload's denoising pass: one layer of the backbone over
    one batch row (two with guidance: the conditional row and its unconditional twin), then the final norm, the LM
    head over that row's masked positions and the unmasking, from the block's first step (every position masked).
    Per-token work is that of the full workload (same hidden size, experts, prefix, vocabulary); a full pass is
    estimated as layers x rows of the layer part plus rows x the head part, the split between the two measured
    once at set-up."""

    def __init__(self, w):
        from block_diffusion_moe_dllm_b200 import synth
        from oracle import dllm_oracle as O
        t0 = time.time()
        self.O = O
        self.w = w
        self.rows = 1 + w.cfg
        self.ws = scaled(w, name=w.name + "-sample", n_layers=1, B=self.rows)
        self.wt = synth.make_weights(self.ws, "cpu")
        caches = synth.make_prefix_cache(self.ws, "cpu")
        tokens, mask = synth.make_block_state(self.ws, "cpu")
        self.hc = [(c[0][:, :, : w.P], c[1][:, :, : w.P]) for c in caches]
        self.tok, self.mask = tokens.numpy(), mask.numpy()
        self.keep = O.sprint_keep(self.ws, self.hc) if w.sprint else None
        a = time.time()
        O.forward_block(self.ws, self.wt, self.hc, self.tok, self.mask, keep=self.keep, want_logits=False)
        b = time.time()
        O.denoise_step(self.ws, self.wt, self.hc, self.tok, self.mask, 0, keep=self.keep)
        c = time.time()
        self.head_frac = min(max(0.0, 1.0 - (b - a) / (c - b)), 1.0)
        self.setup_s = time.time() - t0
        self.cores = len(os.sched_getaffinity(0))

    def step(self):
        """One timed sample; returns (seconds, estimated seconds of one full denoising pass)."""
        a = time.time()
        self.O.denoise_step(self.ws, self.wt, self.hc, self.tok, self.mask, 0, keep=self.keep)
        t = time.time() - a
        w = self.w
        scale_rows = (w.B // self.rows)
        est = t * scale_rows * (w.n_layers * (1.0 - self.head_frac) + self.head_frac)
        return t, est

    def describe(self, n):
        return (f"{n} sample(s) of one layer x {self.rows} batch row(s) x {self.w.L} tokens plus the LM head "
                f"({self.w.vlen} rows) and unmasking of that row, fp64 numpy (BLAS over {self.cores} threads); a "
                f"pass is estimated as {self.w.n_layers} layers x {self.w.B // self.rows} row groups of the layer "
                f"part ({100 * (1 - self.head_frac):.0f}% of the sample) plus {self.w.B // self.rows} x the head "
                f"part; set-up {self.setup_s:.1f}s excluded")


def cpu_baseline(w):
    s = OracleSample(w)
    t, est = s.step()
    return {"value": w.B * w.L / est, "unit": "tokens/s", "cores": s.cores, "kind": "oracle",
            "sample": s.describe(1), "sample_s": t, "pass_s_estimated": est}


# ---------------------------------------------------------------------------------------------- reference arm
def run_reference(args, w):
    _, rank, _ = dist_env()
    if rank != 0:
        return
    s = OracleSample(w)
    for _ in range(args.warmup):
        s.step()
    res = [s.step() for _ in range(args.steps)]
    sample_s = statistics.median(r[0] for r in res)
    est = statistics.median(r[1] for r in res)
    v = w.B * w.L / est
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * sample_s, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "step": "one oracle sample (see cpu_baseline.sample); value = B * L tokens over the estimated time of "
                    "one full denoising pass",
            "config": bench_config(w, args.gpus),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": s.cores, "kind": "oracle",
                             "sample": s.describe(args.steps), "pass_s_estimated": est},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------- block statistics
def block_stats(eng, w, tokens0, mask0):
    """One block decoded pass by pass from the bench's start state (the same kernels and inputs as the timed graph,
    so the same decisions): for each pass, whether it ran, the masked rows it scored and every layer's routed
    experts; the commit pass's routing too."""
    import torch
    eng.set_block(tokens0, mask0)
    E, nl = w.E, w.n_layers
    passes = []
    v = eng.views()

    def counts():
        return eng.expert_counts(v).cpu()

    for t in range(w.T_s):
        n_masked = int(eng.mask[: w.B // (1 + w.cfg)].sum().item())
        eng.step(t)
        torch.cuda.synchronize()
        live = n_masked > 0
        passes.append({"t": t, "live": live, "rows": n_masked,
                       "active": [int((c[:E] > 0).sum()) for c in counts()] if live else None})
    eng.commit()
    torch.cuda.synchronize()
    commit_active = [int((c[:E] > 0).sum()) for c in counts()[: nl - 1]]
    return passes, commit_active


def algorithmic_bytes(w, passes, commit_active):
    """Bytes a block must move at least once from HBM: every live pass reads each layer's attention and router
    weights, the weights of every expert it routed to plus the shared expert, the K/V it attends over, and the
    LM-head rows it scores; SPRINT re-reads the full prefix K and writes the thinned copies at the first pass; the
    commit pass reads the layer weights again (the last layer without its FFN). FP8 expert and LM-head weights
    count one byte per weight plus their row scales. Activations (a few MB) are left out."""
    H, QD = w.H, w.Hq * w.d
    wb = 1 if w.wfmt == "fp8" else 2            # FP8 checkpoint: one byte per expert / LM-head weight (+ row scales)
    attn_w = ((w.Hq + 2 * w.Hkv) * w.d * H + H * QD + w.E * H) * 2
    expert_w = 3 * w.I * H * wb + ((2 * w.I + H) * 4 if wb == 1 else 0)   # gate/up and down row scales
    n_keys = (w.n_keep if w.sprint else w.P) + w.L
    kv = 2 * w.B * w.Hkv * n_keys * w.d * 2
    head = w.vlen * H * wb + (w.vlen * 4 if wb == 1 else 0)
    total = 0
    for p in passes:
        if not p["live"]:
            continue
        for a in p["active"]:
            total += attn_w + (a + 1) * expert_w + kv
        total += head
        if w.sprint and p["t"] == 0:
            total += w.n_layers * w.B * w.Hkv * (w.P + 2 * 2 * w.n_keep) * w.d * 2
    for a in commit_active:
        total += attn_w + (a + 1) * expert_w + kv
    total += attn_w + kv       # the last layer of the commit pass: attention only
    return total


# ---------------------------------------------------------------------------------------------- native arm
def measure(args, w, wt, caches, tokens0, mask0, dev, world, local, e2e):
    """Time whole blocks of workload w through the library's block graph (see the module docstring); with e2e also
    the two end-to-end variants through host buffers. Returns the numbers of the bench line."""
    import torch
    import torch.distributed as dist
    from block_diffusion_moe_dllm_b200 import binding as bd
    from block_diffusion_moe_dllm_b200 import kernel_bench as kb
    from block_diffusion_moe_dllm_b200 import replicas
    from block_diffusion_moe_dllm_b200.engine import DenoiseEngine

    eng = DenoiseEngine(w, wt, caches, dev)
    stream = torch.cuda.current_stream()
    # the whole block as the library's block graph: the T_s passes, each inside a conditional node that runs it only
    # while the block has masked positions, and the commit pass; every step resets the block state from a device
    # copy first. Kernels per pass are counted on host-driven calls.
    eng.set_block(tokens0, mask0)
    eng.decode_block()                      # warms the library's one-time set-up outside capture
    torch.cuda.synchronize()
    n0 = bd.launch_count()
    eng.set_block(tokens0, mask0)
    eng.step(0)
    per_pass = bd.launch_count() - n0
    n0 = bd.launch_count()
    eng.commit()
    per_commit = bd.launch_count() - n0
    graph = eng.block_graph()
    graph_cond = graph.conditional
    graph_note = graph.note

    def block():
        eng.tokens.copy_(tokens0)
        eng.mask.copy_(mask0)
        graph.launch(stream)

    for _ in range(args.warmup):
        block()
    torch.cuda.synchronize()
    assert bd.status_check(eng.ws) == bd.OK

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    units = []
    while not units or (sum(units) < MIN_TIMED_S and len(units) < 50):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            block()
        ev1.record(stream)
        torch.cuda.synchronize()
        units.append(replicas.max_over_ranks(ev0.elapsed_time(ev1) / 1000.0, dev))
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    elapsed = statistics.median(units)
    assert bd.status_check(eng.ws) == bd.OK

    passes, commit_active = block_stats(eng, w, tokens0, mask0)
    live = sum(p["live"] for p in passes)
    Bl = w.B // (1 + w.cfg)
    value = replicas.aggregate_throughput(w.B * w.L * live * args.steps, elapsed, world)
    committed = replicas.aggregate_throughput(Bl * w.L * args.steps, elapsed, world)
    block_bytes = algorithmic_bytes(w, passes, commit_active)
    hbm, hbm_src = kb.hbm_peak()
    step_s = elapsed / args.steps
    act = [a for p in passes if p["live"] for a in p["active"]]
    step_roof = {"bound": "hbm", "algorithmic_bytes": block_bytes, "achieved": block_bytes / step_s / 1e9,
                 "peak": hbm, "unit": "GB/s", "frac": block_bytes / step_s / 1e9 / hbm,
                 "frac_of_spec_8TBs": block_bytes / step_s / 1e9 / SPEC_HBM_GBS,
                 "peak_source": f"{hbm_src} (MEASURED_PEAKS.json hbm_gbs, burst copy)" if hbm_src == "measured"
                 else f"{hbm_src} (profiling recipe figure)"}

    # ---- end to end through the public API with host buffers: every step copies the block state in from pinned
    # host memory, calls dllm_denoise_step for each pass and the commit pass from the host (argument validation,
    # tensor-map encoding and launches included), and copies the final tokens out
    h_tok = tokens0.cpu().pin_memory()
    h_mask = mask0.cpu().pin_memory()
    h_out = torch.empty_like(h_tok).pin_memory()

    def e2e_run(use_graph):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            eng.tokens.copy_(h_tok, non_blocking=True)
            eng.mask.copy_(h_mask, non_blocking=True)
            if use_graph:
                graph.launch(stream)
            else:
                eng.decode_block(stream)
            h_out.copy_(eng.tokens, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        t = replicas.max_over_ranks(e0.elapsed_time(e1) / 1000.0, dev)
        return replicas.aggregate_throughput(w.B * w.L * live * args.steps, t, world)

    io = {"h2d_bytes_per_step": h_tok.numel() * 4 + h_mask.numel(), "d2h_bytes_per_step": h_out.numel() * 4}
    e2e_host = e2e_graph = None
    if e2e:
        e2e_host = {"value": e2e_run(False), "unit": "tokens/s", **io,
                    "path": "dllm_denoise_step called from the host for every pass and the commit pass"}
        e2e_graph = {"value": e2e_run(True), "unit": "tokens/s", **io,
                     "path": "dllm_block_graph_launch per block (passes after the block finished are skipped)"}
    assert bd.status_check(eng.ws) == bd.OK
    del graph
    return {"value": value, "ms_per_step": 1000.0 * step_s, "committed": committed,
            "timed_units": {"n": len(units), "unit_s": units, "steps_per_unit": args.steps},
            "graph_conditional": graph_cond if graph_cond else f"no: {graph_note}",
            "passes_per_block": {"live": live, "launched": live if graph_cond else w.T_s,
                                 "rows_per_live_pass": [p["rows"] for p in passes if p["live"]]},
            "active": {"mean": statistics.mean(act) if act else 0, "min": min(act) if act else 0,
                       "max": max(act) if act else 0},
            "gpu_launches": ((live if graph_cond else w.T_s) * per_pass + per_commit) * args.steps * len(units),
            "clocks": clk, "e2e": e2e_host, "e2e_graph": e2e_graph, "step_roof": step_roof}


def main():
    args = parse()
    w = BY_NAME[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
        return
    import torch
    import torch.distributed as dist
    from block_diffusion_moe_dllm_b200 import binding as bd
    from block_diffusion_moe_dllm_b200 import replicas, synth

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    bd.load()

    seed = replicas.replica_seed(w.seed, rank)
    wt = synth.make_weights(w, dev, seed=seed)
    caches = synth.make_prefix_cache(w, dev, seed=seed)
    tokens0, mask0 = synth.make_block_state(w, dev, seed=seed)
    r = measure(args, w, wt, caches, tokens0, mask0, dev, world, local, e2e=True)

    # ---- the same workload from the FP8 checkpoint (E4M3 expert and LM-head weights with per-row scales): its own
    # routing and passes, since the dequantised weights differ from the bf16 ones
    fp8 = None
    w8 = BY_NAME.get(w.name + "-fp8")
    if w8 is not None and w.wfmt != "fp8" and not args.no_fp8:
        wt8 = synth.make_weights(w8, dev, seed=seed)
        r8 = measure(args, w8, wt8, caches, tokens0, mask0, dev, world, local, e2e=False)
        fp8 = {"workload": w8.name, "value": r8["value"], "unit": "tokens/s", "ms_per_step": r8["ms_per_step"],
               "committed_tokens_per_s": r8["committed"], "passes_per_block": r8["passes_per_block"],
               "active_experts_per_layer": r8["active"], "step_roofline": r8["step_roof"],
               "timed_units": r8["timed_units"], "clocks": r8["clocks"], "gpu_launches": r8["gpu_launches"]}
        del wt8
        torch.cuda.empty_cache()

    # ---- dominant kernel, timed alone with CUDA events at this workload's shapes
    roof, kernels = kernel_rooflines(w, wt, dev, torch.cuda.current_stream())

    if rank == 0:
        line = {"metric": METRIC, "value": r["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "step": "one block: state reset, then the library's block graph: T_s denoising passes, each in a "
                        "conditional node that runs it only while masked positions are left, and the commit pass",
                "config": bench_config(w, world),
                "timed_units": r["timed_units"],
                "committed_tokens_per_s": r["committed"],
                "block_graph_conditional": r["graph_conditional"],
                "passes_per_block": r["passes_per_block"],
                "active_experts_per_layer": r["active"],
                "gpu_launches": r["gpu_launches"],
                "clocks": r["clocks"],
                "e2e": r["e2e"], "e2e_graph": r["e2e_graph"], "roofline": roof, "step_roofline": r["step_roof"],
                "kernels": kernels}
        if fp8 is not None:
            line["fp8_weights"] = fp8
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the roofline kernel from the ncu capture
# summarised in profiles/, keyed by the SHA-256 of the kernel source it was taken with (null once the source changed).
# dram__bytes_read.sum + dram__bytes_write.sum of one launch from an ncu capture of the roofline kernel, valid only for
# the kernel source it was taken with (profiles/gemm_tc_kernel_experts_understanding_512tok.md)
ROOF_TRAFFIC = {"gemm_tc_kernel[experts_swiglu]": {"bytes": 987832832 + 4631296, "sha256": "43ee37f72948904e0272652ef68cba3de62f854a2b64e52cf7c6bbf71cd6a059"}}


def _kernel_traffic(key):
    import hashlib
    entry = ROOF_TRAFFIC.get(key)
    if not entry:
        return None
    src = os.path.join(ROOT, "block_diffusion_moe_dllm_b200", "csrc", "gemm_tc.cu")
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    return entry["bytes"] if sha == entry["sha256"] else None


def kernel_rooflines(w, wt, dev, stream):
    """Per-kernel CUDA-event timings of the step's main calls launched alone at the workload's shapes (a CUDA
    graph of repeated launches). The roofline kernel is the one that moves the most bytes per pass: the SwiGLU
    expert GEMM (gemm_tc_kernel streaming the gate|up weights of every routed expert) when experts dominate, else
    the LM-head GEMM."""
    from block_diffusion_moe_dllm_b200 import kernel_bench as kb
    rows = [kb.bench_lm_head(w, 20, dev, stream, weights=wt)] + kb.bench_proj(w, 20, dev, stream, weights=wt) + \
        kb.bench_experts(w, 20, dev, stream, weights=wt) + kb.bench_expert_gemms(w, 20, dev, stream, weights=wt) + \
        [kb.bench_unmask(w, 20, dev, stream), kb.bench_attn(w, 20, dev, stream)]
    kernels = {r["kernel"]: {k: v for k, v in r.items() if k != "kernel"} for r in rows}
    lm = kernels["gemm_tc_kernel[lm_head]"]
    sw = kernels.get("gemm_tc_kernel[experts_swiglu]")
    name, r = ("gemm_tc_kernel[experts_swiglu]", sw) if sw and sw["bytes"] > lm["bytes"] else \
        ("gemm_tc_kernel[lm_head]", lm)
    roof = {"kernel": name, "bound": "hbm", "achieved": r["GB/s"], "peak": r["peak_GBs"], "unit": "GB/s",
            "frac": r["frac_hbm"], "frac_of_spec_8TBs": r["GB/s"] / SPEC_HBM_GBS, "traffic": _kernel_traffic(name),
            "algorithmic_bytes": r["bytes"], "us_per_launch": r["us"],
            "peak_source": f"{r['peak_source']} (MEASURED_PEAKS.json hbm_gbs, burst copy)"
            if r["peak_source"] == "measured" else f"{r['peak_source']} (profiling recipe figure)"}
    return roof, kernels


if __name__ == "__main__":
    main()
