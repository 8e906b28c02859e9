"""Benchmark of the block-diffusion denoising step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

One bench step decodes one block of the one-layer bf16 workload (hidden 2048, 16 q heads x 128, 4 kv heads,
256 experts top-8 + shared, inter 512, vocab 157184, prefix 1024, block 32, 8 steps): its T_s denoising passes
(embedding, attention over the cached prefix, MoE FFN, LM head over the still-masked rows, confidence +
unmasking) and the commit pass that writes the block's clean K/V into the cache. The block state is reset from a
device copy at the start of every step. metric = denoise-step tokens/s = B * L * T_s tokens through the
denoising passes per second (the commit pass is inside the timed region and not counted). Weights (about 3 GB
streamed, 1.7 GB per pass) exceed the 126 MB L2, so no flush is needed between iterations.

With N > 1 (torchrun), every rank decodes its own replica (independent requests, no collective on the data
path): value = tokens of all ranks / max over ranks of the timed region.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_diffusion_moe_dllm_b200.configs import BY_NAME, ONE_LAYER  # noqa: E402

METRIC = "denoise-step tokens/s (bf16, 1 B200)"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=ONE_LAYER.name)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def dist_env():
    from block_diffusion_moe_dllm_b200 import replicas
    return replicas.env()


# ---------------------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_rank{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
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
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------------- CPU baseline
class OracleRun:
    """The fp64 oracle of the same workload on the host cores (inputs drawn once, on the CPU)."""

    def __init__(self, w):
        from block_diffusion_moe_dllm_b200 import synth
        t0 = time.time()
        self.w = w
        self.wt = synth.make_weights(w, "cpu")
        caches = synth.make_prefix_cache(w, "cpu")
        tokens, mask = synth.make_block_state(w, "cpu")
        self.hc = [(c[0][:, :, : w.P], c[1][:, :, : w.P]) for c in caches]
        self.tok0, self.mask0 = tokens.numpy(), mask.numpy()
        self.setup_s = time.time() - t0

    def run(self, budget_s):
        """Denoising passes from the block's first step until about budget_s seconds of CPU work."""
        from oracle import dllm_oracle as O
        w = self.w
        tok, msk = self.tok0, self.mask0
        passes, t_run, t = 0, 0.0, 0
        while (passes == 0 or t_run < budget_s) and t < w.T_s:
            a = time.time()
            u = O.denoise_step(w, self.wt, self.hc, tok, msk, t)
            t_run += time.time() - a
            tok, msk = u["tokens"], u["mask"]
            passes += 1
            t += 1
        cores = len(os.sched_getaffinity(0))
        return {"value": passes * w.B * w.L / t_run, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                "sample": f"{passes} denoising pass(es) of {w.name} from step 0 (fp64 numpy, BLAS over {cores} "
                          f"threads); input setup {self.setup_s:.1f}s excluded"}


def cpu_baseline(w, budget_s=20.0):
    return OracleRun(w).run(budget_s)


# ---------------------------------------------------------------------------------------------- reference arm
def run_reference(args, w):
    ws_, rank, _ = dist_env()
    if rank != 0:
        return
    orc = OracleRun(w)
    budget = max(2.0, 120.0 / max(args.steps + args.warmup, 1))
    for _ in range(args.warmup):
        orc.run(0.0)
    vals = [orc.run(budget) for _ in range(args.steps)]
    v = statistics.median([x["value"] for x in vals])
    ms = 1000.0 * w.B * w.L * w.T_s / v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "L": w.L, "T_s": w.T_s, "P": w.P},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": vals[0]["cores"], "kind": "oracle",
                             "sample": vals[0]["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------- native arm
def main():
    args = parse()
    w = BY_NAME[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
        return
    import torch
    import torch.distributed as dist
    from block_diffusion_moe_dllm_b200 import binding as bd
    from block_diffusion_moe_dllm_b200 import synth
    from block_diffusion_moe_dllm_b200.engine import DenoiseEngine

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    bd.load()

    from block_diffusion_moe_dllm_b200 import replicas
    seed = replicas.replica_seed(w.seed, rank)
    wt = synth.make_weights(w, dev, seed=seed)
    caches = synth.make_prefix_cache(w, dev, seed=seed)
    tokens0, mask0 = synth.make_block_state(w, dev, seed=seed)
    eng = DenoiseEngine(w, wt, caches, dev)
    stream = torch.cuda.current_stream()

    # the whole block (state reset + T_s passes + commit) as one CUDA graph; the library's launches per block are
    # counted while it is captured
    n0 = bd.launch_count()
    g_reset = eng.capture_block(tokens0, mask0)
    launches_per_step = (bd.launch_count() - n0) // 3      # two warm-up blocks + the captured one
    g_plain = eng.capture_block()                           # the same without the device-side reset (e2e arm)

    for _ in range(args.warmup):
        g_reset.replay()
    torch.cuda.synchronize()
    assert bd.status_check(eng.ws) == bd.OK

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        g_reset.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    launches = launches_per_step * args.steps
    elapsed = replicas.max_over_ranks(ev0.elapsed_time(ev1) / 1000.0, dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    tokens_per_step = w.B * w.L * w.T_s
    value = replicas.aggregate_throughput(tokens_per_step * args.steps, elapsed, world)

    # ---- end to end through the public API with host buffers: block state from pinned host memory in,
    # final tokens out, every step
    h_tok = tokens0.cpu().pin_memory()
    h_mask = mask0.cpu().pin_memory()
    h_out = torch.empty_like(h_tok).pin_memory()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        eng.tokens.copy_(h_tok, non_blocking=True)
        eng.mask.copy_(h_mask, non_blocking=True)
        g_plain.replay()
        h_out.copy_(eng.tokens, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_t = replicas.max_over_ranks(e0.elapsed_time(e1) / 1000.0, dev)
    e2e = {"value": replicas.aggregate_throughput(tokens_per_step * args.steps, e2e_t, world), "unit": "tokens/s",
           "h2d_bytes_per_step": h_tok.numel() * 4 + h_mask.numel(), "d2h_bytes_per_step": h_out.numel() * 4}
    del g_reset, g_plain

    # ---- dominant kernel, timed alone with CUDA events: the tensor-core GEMM streaming the LM head
    # (157184 x 2048 bf16) for the 32 masked rows of the first pass
    roof, kernels = kernel_rooflines(w, wt, eng, dev, stream)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": 1000.0 * elapsed / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": w.name, "B": w.B, "L": w.L, "T_s": w.T_s, "P": w.P, "H": w.H, "E": w.E,
                           "k": w.k, "I": w.I, "V": w.V, "layers": w.n_layers,
                           "parallelism": f"replicas{world}" if world > 1 else "single",
                           "l2": "inputs larger than L2 (weights streamed per pass)",
                           "step": "one block: T_s denoising passes + commit pass, replayed as one CUDA graph"},
                "gpu_launches": launches, "clocks": clk, "e2e": e2e, "roofline": roof, "kernels": kernels}
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one LM-head launch of gemm_tc_kernel from the ncu
# capture summarised in profiles/, keyed by the SHA-256 of the kernel source it was taken with.
LM_HEAD_TRAFFIC = {"sha256": "31452c4b1d34db9acb4517560a598dacc90f73b2d9cc49c7677e9fcbb9ce2179", "bytes": 644.037120e6 + 6.460672e6}


def _kernel_traffic():
    import hashlib
    src = os.path.join(ROOT, "block_diffusion_moe_dllm_b200", "csrc", "gemm_tc.cu")
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    return LM_HEAD_TRAFFIC["bytes"] if sha == LM_HEAD_TRAFFIC["sha256"] else None


def kernel_rooflines(w, wt, eng, dev, stream):
    """Per-kernel CUDA-event timings of the step's main calls launched alone with the step's shapes; the LM-head
    GEMM (one launch of gemm_tc_kernel streaming 157184 x 2048 bf16) is the roofline kernel."""
    from block_diffusion_moe_dllm_b200 import kernel_bench as kb
    lm = kb.bench_lm_head(w, 20, dev, stream, weights=wt)
    rest = (kb.bench_proj(w, 20, dev, stream, weights=wt) + kb.bench_experts(w, 20, dev, stream, weights=wt) +
            [kb.bench_unmask(w, 20, dev, stream), kb.bench_attn(w, 20, dev, stream)])
    kernels = {r["kernel"]: {k: v for k, v in r.items() if k != "kernel"} for r in [lm] + rest}
    roof = {"kernel": "gemm_tc_kernel (LM head 157184x2048 bf16, 32 rows)", "bound": "hbm",
            "achieved": lm["GB/s"], "peak": lm["peak_GBs"], "unit": "GB/s", "frac": lm["frac_hbm"],
            "traffic": _kernel_traffic(), "algorithmic_bytes": lm["bytes"],
            "peak_source": f"{lm['peak_source']} (MEASURED_PEAKS.json hbm_gbs, burst copy)"}
    return roof, kernels


if __name__ == "__main__":
    main()
