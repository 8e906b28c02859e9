"""Seeded synthetic inputs for the denoising step (weights, caches, block state, logits).

This module only draws random numbers; it holds none of the method's arithmetic. Every tensor is drawn from
torch's generator seeded by (seed, tag), on the device asked for, so a workload is reproducible. The values are
stored in the workload's storage type (bf16 round-to-nearest-even from the fp32 draw, or fp32).

Recipe (weights of an untrained backbone of the stated architecture):
  projection, router, expert and LM-head matrices ~ N(0, w_std^2)   (LM head: N(0, lm_std^2))
  router bias ~ U(-bias_range, bias_range)                            (fp32)
  embedding rows ~ N(0, 1)
  RMSNorm gains = 1 (or ~ U(0.5, 1.5) when ``random_gains``)
  prefix K/V cache ~ N(0, 1)
  block tokens ~ U[0, V - 1), every position masked at the first step
"""
import zlib
import torch

from .configs import Workload

_TORCH_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def torch_dtype(name: str) -> torch.dtype:
    return _TORCH_DT[name]


def _gen(seed: int, tag: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + zlib.crc32(tag.encode())) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def normal(shape, std, seed, tag, device="cpu", dtype=torch.bfloat16, chunk_rows=None):
    """N(0, std^2) draw, rounded to ``dtype``. Large tensors are drawn in row chunks to bound fp32 scratch."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=dtype, device=device)
    g = _gen(seed, tag, device)
    if chunk_rows is None or shape[0] <= chunk_rows:
        out.copy_(torch.randn(shape, generator=g, device=device, dtype=torch.float32).mul_(std))
    else:
        for r0 in range(0, shape[0], chunk_rows):
            r1 = min(shape[0], r0 + chunk_rows)
            out[r0:r1].copy_(torch.randn((r1 - r0,) + shape[1:], generator=g, device=device,
                                         dtype=torch.float32).mul_(std))
    return out


def uniform(shape, lo, hi, seed, tag, device="cpu", dtype=torch.float32):
    g = _gen(seed, tag, device)
    x = torch.rand(tuple(shape), generator=g, device=device, dtype=torch.float32)
    return (x * (hi - lo) + lo).to(dtype)


def randint(shape, lo, hi, seed, tag, device="cpu"):
    g = _gen(seed, tag, device)
    return torch.randint(lo, hi, tuple(shape), generator=g, device=device, dtype=torch.int64).to(torch.int32)


def fp8_rows(wb, chunk_rows=16384):
    """An FP8 checkpoint of the bf16 matrix wb [..., M, K]: E4M3 codes (uint8) and one fp32 scale per row,
    scale = max |row| / 448 (1 for an all-zero row), codes = round-to-nearest E4M3 of row / scale (torch's
    float8_e4m3fn conversion), row by row in chunks."""
    shape = wb.shape
    flat = wb.reshape(-1, shape[-1])
    codes = torch.empty(flat.shape, dtype=torch.uint8, device=wb.device)
    scale = torch.empty(flat.shape[0], dtype=torch.float32, device=wb.device)
    for r0 in range(0, flat.shape[0], chunk_rows):
        f = flat[r0: r0 + chunk_rows].float()
        amax = f.abs().amax(dim=1)
        sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
        codes[r0: r0 + chunk_rows] = (f / sc[:, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        scale[r0: r0 + chunk_rows] = sc
    return codes.reshape(shape), scale.reshape(shape[:-1])


def make_weights(w: Workload, device="cpu", seed=None, random_gains=False):
    """All backbone weights of workload ``w``. Returns a dict of tensors on ``device``. With w.wfmt == "fp8" the
    expert and LM-head weights are replaced by their FP8 checkpoint (E4M3 codes, plus "<name>_scale" row scales)."""
    s = w.seed if seed is None else seed
    dt = torch_dtype(w.dtype)
    H, Hq, Hkv, d, E, I, V = w.H, w.Hq, w.Hkv, w.d, w.E, w.I, w.V
    big = 1 << 14

    def gain(tag):
        if random_gains:
            return uniform((H,), 0.5, 1.5, s, tag, device, dt)
        return torch.ones(H, dtype=dt, device=device)

    wt = {
        "embed": normal((V, H), 1.0, s, "embed", device, dt, big),
        "final_norm": gain("final_norm"),
        "w_lm": normal((V, H), w.lm_std, s, "w_lm", device, dt, big),
        "layers": [],
    }
    for l in range(w.n_layers):
        p = f"L{l}."
        wt["layers"].append({
            "attn_norm": gain(p + "attn_norm"),
            "w_qkv": normal(((Hq + 2 * Hkv) * d, H), w.w_std, s, p + "w_qkv", device, dt),
            "w_o": normal((H, Hq * d), w.w_std, s, p + "w_o", device, dt),
            "ffn_norm": gain(p + "ffn_norm"),
            "w_router": normal((E, H), w.w_std, s, p + "w_router", device, dt),
            "router_bias": uniform((E,), -w.bias_range, w.bias_range, s, p + "router_bias", device),
            "w_gu": normal((E, 2 * I, H), w.w_std, s, p + "w_gu", device, dt, 16),
            "w_down": normal((E, H, I), w.w_std, s, p + "w_down", device, dt, 16),
            "w_gu_shared": normal((2 * I, H), w.w_std, s, p + "w_gu_shared", device, dt),
            "w_down_shared": normal((H, I), w.w_std, s, p + "w_down_shared", device, dt),
        })
    if w.wfmt == "fp8":
        wt["w_lm"], wt["w_lm_scale"] = fp8_rows(wt["w_lm"])
        for lw in wt["layers"]:
            for name in ("w_gu", "w_down", "w_gu_shared", "w_down_shared"):
                lw[name], lw[name + "_scale"] = fp8_rows(lw[name])
    return wt


def make_prefix_cache(w: Workload, device="cpu", seed=None, cap=None):
    """Per-layer K and V caches [B, Hkv, cap, d], rows [0, P) filled with N(0,1), the rest zero."""
    s = w.seed if seed is None else seed
    dt = torch_dtype(w.dtype)
    cap = w.cap if cap is None else cap
    caches = []
    for l in range(w.n_layers):
        kc = torch.zeros((w.B, w.Hkv, cap, w.d), dtype=dt, device=device)
        vc = torch.zeros((w.B, w.Hkv, cap, w.d), dtype=dt, device=device)
        if w.P:
            kc[:, :, : w.P].copy_(normal((w.B, w.Hkv, w.P, w.d), 1.0, s, f"L{l}.k_cache", device, dt))
            vc[:, :, : w.P].copy_(normal((w.B, w.Hkv, w.P, w.d), 1.0, s, f"L{l}.v_cache", device, dt))
        caches.append((kc, vc))
    return caches


def make_block_state(w: Workload, device="cpu", seed=None, masked_fraction=1.0):
    """Block tokens [B, L] int32 and mask [B, L] uint8. In guided workloads every row group (halves with cfg 1,
    thirds with cfg 2) shares the first group's pattern."""
    s = w.seed if seed is None else seed
    tokens = randint((w.B, w.L), 0, w.V - 1, s, "block_tokens", device)
    if masked_fraction >= 1.0:
        mask = torch.ones((w.B, w.L), dtype=torch.uint8, device=device)
    else:
        u = uniform((w.B, w.L), 0.0, 1.0, s, "block_mask", device)
        mask = (u < masked_fraction).to(torch.uint8)
    if w.cfg:
        Bl = w.B // (1 + w.cfg)
        for g in range(1, 1 + w.cfg):
            mask[g * Bl:(g + 1) * Bl] = mask[:Bl]
            tokens[g * Bl:(g + 1) * Bl] = tokens[:Bl]
    tokens = torch.where(mask.bool(), torch.full_like(tokens, w.mask_id), tokens)
    return tokens, mask


def skewed_expert_choices(rows, E, k, seed, tag="skewed_ids", n_hot=8, n_warm=60, p_hot=0.67):
    """Expert choices [rows, k] int32 (distinct per row) with the skew a block's own router shows on an untrained
    backbone, where most block positions hold the same mask token: each slot picks, with probability ``p_hot``, one
    of ``n_hot`` crowded experts, else one of ``n_warm`` others (both sets drawn at random from the E experts).
    Measured on the 20-layer understanding workload: about 8 experts with 340-512 rows each and some 60 with a
    median of 18 rows take the 4096 assignments of 512 rows."""
    g = _gen(seed, tag, "cpu")
    experts = torch.randperm(E, generator=g)
    hot, warm = experts[:n_hot], experts[n_hot:n_hot + n_warm]
    ids = torch.empty((rows, k), dtype=torch.int32)
    u = torch.rand((rows, k), generator=g)
    for r in range(rows):
        taken = set()
        for j in range(k):
            pool = hot if (u[r, j] < p_hot and len(taken & set(hot.tolist())) < n_hot) else warm
            while True:
                e = int(pool[int(torch.randint(0, len(pool), (1,), generator=g))])
                if e not in taken:
                    break
            taken.add(e)
            ids[r, j] = e
    return ids
