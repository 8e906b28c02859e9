"""Per-call parity of the CUDA library against the fp64 oracle on seeded inputs (GPU)."""
import ctypes as C
import math

import numpy as np
import pytest
import torch

from block_diffusion_moe_dllm_b200 import binding as bd
from block_diffusion_moe_dllm_b200 import synth
from oracle import dllm_oracle as O
from _util import ROUTE_TIE, TOL, assert_close, assignment_tables, check_unmask, random_assignments, same_routing, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
DT = {"bf16": bd.BF16, "f32": bd.F32}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    bd.load()


def _tdt(name):
    return synth.torch_dtype(name)


# ------------------------------------------------------------------------------------------------ GEMM
@pytest.mark.parametrize("N,M,K", [(1, 128, 64), (5, 256, 128), (32, 384, 2048), (77, 256, 512), (200, 128, 256),
                                   (300, 256, 192), (513, 128, 64), (512, 3072, 2048), (500, 3072, 512),
                                   (440, 2816, 1024)])
def test_gemm_bf16_store(N, M, K):
    """Dense projections; the last three take the 96-row N tile (one wave of 96-row tiles where 128-row tiles would
    leave a quarter of the SMs idle), ragged at 500 and 440 rows."""
    x = synth.normal((N, K), 1.0, 1, f"gx{N}", DEV)
    w = synth.normal((M, K), 0.05, 1, f"gw{M}{K}", DEV)
    y = torch.full((N, M), float("nan"), dtype=torch.bfloat16, device=DEV)
    bd.gemm(x, w, y, N, M, K, bd.BF16)
    torch.cuda.synchronize()
    want = O.store(to64(x) @ to64(w).T, "bf16")
    assert_close(to64(y), want, "bf16", "gemm")


@pytest.mark.parametrize("N,M,K", [(32, 3072, 2048), (32, 2048, 2048), (7, 256, 1024),
                                   (512, 256, 2048), (77, 256, 512), (100, 512, 1024)])
def test_gemm_bf16_split_k(N, M, K):
    """Few output tiles: the K slices of a tile run as one thread-block cluster and are summed through distributed
    shared memory (one or several 32-row N tiles, ragged last tile)."""
    x = synth.normal((N, K), 1.0, 9, f"skx{N}", DEV)
    w = synth.normal((M, K), 0.02, 9, f"skw{M}", DEV)
    y0 = synth.normal((N, M), 1.0, 9, f"sky{N}{M}", DEV)
    y = y0.clone()
    bd.gemm(x, w, y, N, M, K, bd.BF16, residual=1)
    torch.cuda.synchronize()
    assert_close(to64(y), O.store(to64(y0) + to64(x) @ to64(w).T, "bf16"), "bf16", "split-K gemm")


@pytest.mark.parametrize("N,M,K,residual", [(512, 256, 2048, 0), (300, 512, 1024, 1), (384, 384, 2048, 1),
                                            (1000, 512, 2048, 0)])
def test_gemm_bf16_wide_split_k(N, M, K, residual):
    """A block's rows (hundreds) against a projection of at most four weight tiles (the router's logits): N tiles
    of 128 rows (256 at 1000 rows) whose eight K slices run as one cluster, every slice's accumulator staged in its
    operand ring and each rank reducing and storing its share of the columns (ragged last N tiles at 300 and 1000
    rows)."""
    x = synth.normal((N, K), 1.0, 12, f"wx{N}{K}", DEV)
    w = synth.normal((M, K), 0.02, 12, f"ww{M}{K}", DEV)
    y0 = synth.normal((N, M), 1.0, 12, f"wy{N}{M}", DEV)
    y = y0.clone()
    bd.gemm(x, w, y, N, M, K, bd.BF16, residual=residual)
    torch.cuda.synchronize()
    acc = to64(x) @ to64(w).T
    want = O.store(to64(y0) + acc, "bf16") if residual else O.store(acc, "bf16")
    assert_close(to64(y), want, "bf16", "gemm (wide split-K)")


@pytest.mark.parametrize("N,M,K,residual", [(1200, 2048, 256, 0), (4100, 2048, 512, 1), (600, 4096, 128, 0)])
def test_gemm_bf16_cta_pairs(N, M, K, residual):
    """N tile 256 with enough tiles: CTA pairs share each MMA (M = 256 across two SMs, half of the N tile's rows
    from each); ragged last N tiles (176, 4 and 88 rows)."""
    x = synth.normal((N, K), 1.0, 10, f"px{N}", DEV)
    w = synth.normal((M, K), 0.05, 10, f"pw{M}{K}", DEV)
    y0 = synth.normal((N, M), 1.0, 10, f"py{N}{M}", DEV)
    y = y0.clone()
    bd.gemm(x, w, y, N, M, K, bd.BF16, residual=residual)
    torch.cuda.synchronize()
    acc = to64(x) @ to64(w).T
    want = O.store(to64(y0) + acc, "bf16") if residual else O.store(acc, "bf16")
    assert_close(to64(y), want, "bf16", "gemm (CTA pairs)")


def test_gemm_bf16_residual_and_device_count():
    N, M, K = 40, 256, 256
    x = synth.normal((N, K), 1.0, 2, "rx", DEV)
    w = synth.normal((M, K), 0.05, 2, "rw", DEV)
    y0 = synth.normal((N, M), 1.0, 2, "ry", DEV)
    y = y0.clone()
    n_dev = torch.tensor([33], dtype=torch.int32, device=DEV)
    bd.gemm(x, w, y, N, M, K, bd.BF16, residual=1, n_rows_dev=n_dev)
    torch.cuda.synchronize()
    want = O.store(to64(y0)[:33] + to64(x)[:33] @ to64(w).T, "bf16")
    assert_close(to64(y)[:33], want, "bf16", "gemm residual")
    assert torch.equal(y[33:], y0[33:]), "rows past the device count must be untouched"


def test_gemm_bf16_f32_output():
    N, M, K = 17, 128, 320
    x = synth.normal((N, K), 1.0, 3, "fx", DEV)
    w = synth.normal((M, K), 0.05, 3, "fw", DEV)
    y = torch.zeros((N, M), dtype=torch.float32, device=DEV)
    bd.gemm(x, w, y, N, M, K, bd.BF16, y_f32=1)
    torch.cuda.synchronize()
    want = to64(x) @ to64(w).T
    assert np.max(np.abs(to64(y) - want)) < 1e-4


def test_gemm_f32():
    N, M, K = 23, 100, 70
    x = synth.normal((N, K), 1.0, 4, "sx", DEV, torch.float32)
    w = synth.normal((M, K), 0.05, 4, "sw", DEV, torch.float32)
    y = torch.zeros((N, M), dtype=torch.float32, device=DEV)
    bd.gemm(x, w, y, N, M, K, bd.F32)
    torch.cuda.synchronize()
    assert_close(to64(y), to64(x) @ to64(w).T, "f32", "gemm f32")


# ------------------------------------------------------------------------------------------------ router
@pytest.mark.parametrize("dtype,Tk,H,E,k", [("bf16", 1, 2048, 256, 8), ("bf16", 32, 2048, 256, 8),
                                            ("bf16", 77, 2048, 256, 8), ("bf16", 512, 2048, 256, 8),
                                            ("f32", 16, 256, 8, 2), ("bf16", 9, 256, 1024, 32),
                                            ("bf16", 20, 256, 512, 8), ("f32", 32, 128, 64, 32),
                                            ("bf16", 4096, 512, 256, 8), ("bf16", 1001, 256, 1000, 3),
                                            ("f32", 4100, 64, 32, 2), ("bf16", 5000, 256, 96, 4),
                                            ("bf16", 1024, 512, 128, 8), ("f32", 4096, 64, 32, 2),
                                            ("bf16", 33, 256, 96, 4), ("f32", 1000, 128, 200, 6)])
def test_route(dtype, Tk, H, E, k):
    t = _tdt(dtype)
    h = synth.normal((Tk, H), 1.0, 5, f"rh{Tk}", DEV, t)
    wr = synth.normal((E, H), 0.02, 5, f"rw{E}", DEV, t)
    bias = synth.uniform((E,), -0.1, 0.1, 5, f"rb{E}", DEV)
    ids = torch.empty((Tk, k), dtype=torch.int32, device=DEV)
    gates = torch.empty((Tk, k), dtype=torch.float32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(Tk * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(Tk * k, dtype=torch.int32, device=DEV)
    scores = torch.empty((Tk, E), dtype=torch.float32, device=DEV)
    bd.moe_route(h, wr, bias, ids, gates, counts, offsets, perm, inv, Tk, H, E, k, DT[dtype], scores=scores)
    torch.cuda.synchronize()
    o_ids, o_gates, o_s, margin = O.route(to64(h), to64(wr), to64(bias), k, order=True)
    g_ids = ids.cpu().numpy()
    # the fp32 scores stay well inside the library's re-decision guard (2e-5 between neighbours)
    assert np.max(np.abs(to64(scores) - o_s)) < 2e-6
    same_routing(g_ids, gates.cpu().numpy(), o_ids, o_gates, margin >= ROUTE_TIE, rtol=2e-6, atol=2e-7)
    # permutation tables are exactly those of the GPU's ids
    c, off, p, iv = assignment_tables(g_ids, E)
    assert np.array_equal(counts.cpu().numpy(), c)
    assert np.array_equal(offsets.cpu().numpy(), off)
    assert np.array_equal(perm.cpu().numpy(), p)
    assert np.array_equal(inv.cpu().numpy(), iv)


@pytest.mark.parametrize("dtype,Tk", [("f32", 2000), ("bf16", 2000), ("bf16", 300)])
def test_route_planted_near_ties(dtype, Tk):
    """Every token's second slot is contested by two experts whose scores differ by 1e-6 .. 1e-5 (inside the
    library's fp32 guard, outside the 1e-6 band the comparison forgives): expert 0 always wins slot 1 (bias 2),
    experts 1 and 2 (bias 1) differ only by a tiny weight perturbation, so nearly every token is re-decided exactly,
    more of them than one CTA's flagged list holds."""
    t = _tdt(dtype)
    H, E, k = 256, 64, 2
    g = torch.Generator().manual_seed(1234)
    h = torch.randn((Tk, H), generator=g, dtype=torch.float64)
    w = torch.randn((E, H), generator=g, dtype=torch.float64) * 0.02
    bias = (torch.rand(E, generator=g, dtype=torch.float64) - 0.5) * 0.2
    bias[0], bias[1], bias[2] = 2.0, 1.0, 1.0
    if dtype == "f32":
        w[2] = w[1] + 1e-6 * torch.randn(H, generator=g, dtype=torch.float64)
        hd, wd = h.to(t), w.to(t)
    else:
        j = 7
        w[1, j] = 0.02
        sgn = torch.where(torch.rand(Tk, generator=g) < 0.5, -1.0, 1.0).to(torch.float64)
        h[:, j] = sgn * (0.04 + 0.26 * torch.rand(Tk, generator=g, dtype=torch.float64))
        hd, wd = h.to(t), w.to(t)
        wb = wd.view(torch.int16)
        wb[2] = wb[1]
        wb[2, j] += 1                      # one bf16 ulp apart in one coordinate
    hd, wd = hd.to(DEV), wd.to(DEV)
    bias_d = bias.to(torch.float32).to(DEV)
    ids = torch.empty((Tk, k), dtype=torch.int32, device=DEV)
    gates = torch.empty((Tk, k), dtype=torch.float32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(Tk * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(Tk * k, dtype=torch.int32, device=DEV)
    bd.moe_route(hd, wd, bias_d, ids, gates, counts, offsets, perm, inv, Tk, H, E, k, DT[dtype])
    torch.cuda.synchronize()
    o_ids, o_gates, _, margin = O.route(to64(hd), to64(wd), to64(bias_d), k, order=True)
    checked = margin >= ROUTE_TIE
    near = checked & (margin < 1e-5)
    assert near.sum() >= min(257, Tk // 3), "the planted ties should put many tokens inside the guard"
    g_ids = ids.cpu().numpy()
    same_routing(g_ids, gates.cpu().numpy(), o_ids, o_gates, checked, rtol=2e-6, atol=2e-7)
    c, off, p, iv = assignment_tables(g_ids, E)
    assert np.array_equal(counts.cpu().numpy(), c)
    assert np.array_equal(offsets.cpu().numpy(), off)
    assert np.array_equal(perm.cpu().numpy(), p)
    assert np.array_equal(inv.cpu().numpy(), iv)


# ------------------------------------------------------------------------------------------------ experts
@pytest.mark.parametrize("dtype,Tk,H,E,k,I,shared", [("bf16", 32, 2048, 256, 8, 512, True),
                                                     ("bf16", 5, 256, 16, 4, 128, True),
                                                     ("bf16", 70, 256, 8, 2, 192, False),
                                                     ("bf16", 300, 256, 4, 2, 64, True),
                                                     ("bf16", 600, 256, 4, 2, 128, True),
                                                     ("f32", 16, 256, 8, 2, 128, True)])
def test_experts(dtype, Tk, H, E, k, I, shared):
    t = _tdt(dtype)
    h = synth.normal((Tk, H), 1.0, 6, "eh", DEV, t)
    x0 = synth.normal((Tk, H), 1.0, 6, "ex", DEV, t)
    wgu = synth.normal((E, 2 * I, H), 0.02, 6, "egu", DEV, t)
    wd = synth.normal((E, H, I), 0.02, 6, "ed", DEV, t)
    sgu = synth.normal((2 * I, H), 0.02, 6, "sgu", DEV, t) if shared else None
    sd = synth.normal((H, I), 0.02, 6, "sd", DEV, t) if shared else None
    ids, gates = random_assignments(Tk, E, k, seed=Tk + E)
    counts, offsets, perm, inv = assignment_tables(ids, E)
    cvt = lambda a: torch.from_numpy(a).to(DEV)
    x = x0.clone()
    bd.moe_experts(h, wgu, wd, sgu, sd, cvt(counts), cvt(offsets), cvt(perm), cvt(inv), cvt(gates), x, Tk, H, E, k,
                   I, DT[dtype])
    torch.cuda.synchronize()
    delta = O.moe_delta(to64(h), ids, gates.astype(np.float64), to64(wgu), to64(wd),
                        to64(sgu) if shared else None, to64(sd) if shared else None, dtype)
    want = O.store(to64(x0) + delta, dtype)
    assert_close(to64(x), want, dtype, "experts")


@pytest.mark.parametrize("Tk", [512, 200])
def test_experts_crowded_routing_with_stale_work_counters(Tk):
    """The block's own routing piles rows on a few experts (synth.skewed_expert_choices: 8 crowded experts with
    hundreds of rows, ~60 with a few each): the tiles the expert GEMMs' dynamic schedule balances. The schedule's
    work counters sit in the workspace's status block and are reset by the row gather at every call, so words left
    there by anything else (planted here) must not change the result."""
    dtype, H, E, k, I = "bf16", 2048, 256, 8, 512
    t = _tdt(dtype)
    h = synth.normal((Tk, H), 1.0, 16, "ch", DEV, t)
    x0 = synth.normal((Tk, H), 1.0, 16, "cx", DEV, t)
    wgu = synth.normal((E, 2 * I, H), 0.02, 16, "cgu", DEV, t)
    wd = synth.normal((E, H, I), 0.02, 16, "cd", DEV, t)
    sgu = synth.normal((2 * I, H), 0.02, 16, "csgu", DEV, t)
    sd = synth.normal((H, I), 0.02, 16, "csd", DEV, t)
    ids = synth.skewed_expert_choices(Tk, E, k, 16).numpy()
    g = np.random.default_rng(Tk)
    gates = g.uniform(0.1, 1.0, (Tk, k)).astype(np.float32)
    gates = (gates / gates.sum(1, keepdims=True)).astype(np.float32)
    counts, offsets, perm, inv = assignment_tables(ids, E)
    assert counts.max() >= 128, "the case must hold experts with more rows than one N tile"
    cvt = lambda a: torch.from_numpy(a).to(DEV)
    desc = bd.ExpertDesc(Tk, H, E, k, I, DT[dtype], 0)
    ws = bd.Workspace(bd.load().dllm_moe_experts_workspace_size(C.byref(desc)), DEV)
    off = ws.addr - ws.buf.data_ptr()
    for word in (16, 32):   # the two GEMMs' counters (bytes 64 and 128 of the status block)
        ws.buf[off + 4 * word: off + 4 * word + 4] = torch.tensor([0x78, 0x56, 0x34, 0x12], dtype=torch.uint8)
    x = x0.clone()
    bd.moe_experts(h, wgu, wd, sgu, sd, cvt(counts), cvt(offsets), cvt(perm), cvt(inv), cvt(gates), x, Tk, H, E, k,
                   I, DT[dtype], ws=ws)
    torch.cuda.synchronize()
    assert bd.status_check(ws) == bd.OK
    delta = O.moe_delta(to64(h), ids, gates.astype(np.float64), to64(wgu), to64(wd), to64(sgu), to64(sd), dtype)
    want = O.store(to64(x0) + delta, dtype)
    assert_close(to64(x), want, dtype, "experts, crowded routing")


@pytest.mark.parametrize("Tk,E,k,I,H,swiglu", [(512, 256, 8, 512, 2048, 1), (512, 256, 8, 512, 2048, 0),
                                                  (77, 16, 4, 128, 256, 1), (300, 8, 2, 128, 256, 0)])
def test_grouped_gemm(Tk, E, k, I, H, swiglu):
    """dllm_grouped_gemm over router-shaped groups plus the shared expert's rows: SwiGLU (gate|up, stored bf16) or the
    down projection (fp32 rows), against the oracle's per-group products (sampled rows of every group)."""
    ids, _ = random_assignments(Tk, E, k, seed=Tk + I)
    counts, offsets, perm, _ = assignment_tables(ids, E)
    n = Tk * k + Tk
    K, M = (H, I) if swiglu else (I, H)
    x = synth.normal((n, K), 1.0, 9, f"gg_x{K}", DEV)
    w = synth.normal((E, 2 * M if swiglu else M, K), 0.02, 9, f"gg_w{M}", DEV)
    wx = synth.normal((2 * M if swiglu else M, K), 0.02, 9, f"gg_s{M}", DEV)
    y = torch.full((n, M), -3.0, dtype=torch.bfloat16 if swiglu else torch.float32, device=DEV)
    cvt = lambda a: torch.from_numpy(a).to(DEV)
    bd.grouped_gemm(x, w, wx, cvt(counts), cvt(offsets[:-1].copy()), y, E, n, K, M, bd.BF16, swiglu=swiglu,
                    extra_rows=Tk, max_rows_hint=max(64, 4 * (Tk * k // E)), y_f32=0 if swiglu else 1)
    torch.cuda.synchronize()
    xs, ys = to64(x), to64(y)
    g = np.random.default_rng(3)
    groups = [(int(offsets[e]), int(counts[e]), to64(w[e])) for e in range(E) if counts[e] > 0]
    groups.append((Tk * k, Tk, to64(wx)))
    for off, cnt, we in groups:
        r = np.unique(g.integers(off, off + cnt, min(cnt, 4)))
        if swiglu:
            gt, up = xs[r] @ we[:M].T, xs[r] @ we[M:].T
            want = O.store(O.silu(gt) * up, "bf16")
            assert_close(ys[r], want, "bf16", "grouped SwiGLU rows")
        else:
            want = xs[r] @ we.T
            assert np.all(np.abs(ys[r] - want) <= 1e-4 * np.maximum(1.0, np.abs(want))), "grouped GEMM rows"


@pytest.mark.parametrize("Tk,E,k,I,H,swiglu", [(512, 256, 8, 512, 2048, 1), (512, 256, 8, 512, 2048, 0),
                                                  (40, 16, 4, 128, 256, 1), (300, 8, 2, 128, 256, 0)])
def test_grouped_gemm_fp8(Tk, E, k, I, H, swiglu):
    """dllm_grouped_gemm with E4M3 weights and per-row scales (the FP8 checkpoint) against the oracle's products
    with the dequantized weights, on sampled rows of every group (N tiles of 32, 64 and 128 rows)."""
    ids, _ = random_assignments(Tk, E, k, seed=Tk + I + 1)
    counts, offsets, perm, _ = assignment_tables(ids, E)
    n = Tk * k + Tk
    K, M = (H, I) if swiglu else (I, H)
    Mw = 2 * M if swiglu else M
    x = synth.normal((n, K), 1.0, 10, f"gf_x{K}", DEV)
    wq, ws_ = synth.fp8_rows(synth.normal((E, Mw, K), 0.02, 10, f"gf_w{M}", DEV))
    xq, xs = synth.fp8_rows(synth.normal((Mw, K), 0.02, 10, f"gf_s{M}", DEV))
    y = torch.full((n, M), -3.0, dtype=torch.bfloat16 if swiglu else torch.float32, device=DEV)
    cvt = lambda a: torch.from_numpy(a).to(DEV)
    bd.grouped_gemm(x, wq, xq, cvt(counts), cvt(offsets[:-1].copy()), y, E, n, K, M, bd.BF16, swiglu=swiglu,
                    extra_rows=Tk, max_rows_hint=max(32, 4 * (Tk * k // E)), y_f32=0 if swiglu else 1, w_scale=ws_,
                    w_extra_scale=xs)
    torch.cuda.synchronize()
    xs64, ys = to64(x), to64(y)
    g = np.random.default_rng(4)
    groups = [(int(offsets[e]), int(counts[e]), e) for e in range(E) if counts[e] > 0] + [(Tk * k, Tk, -1)]
    for off, cnt, e in groups:
        q, sc = (xq, xs) if e < 0 else (wq[e], ws_[e])
        we = O.dequant_rows(q.cpu().numpy(), sc.cpu().numpy())
        r = np.unique(g.integers(off, off + cnt, min(cnt, 4)))
        if swiglu:
            want = O.store(O.silu(xs64[r] @ we[:M].T) * (xs64[r] @ we[M:].T), "bf16")
            assert_close(ys[r], want, "bf16", "grouped SwiGLU rows (FP8 weights)")
        else:
            want = xs64[r] @ we.T
            assert np.all(np.abs(ys[r] - want) <= 1e-4 * np.maximum(1.0, np.abs(want))), "grouped rows (FP8)"


@pytest.mark.parametrize("N", [32, 200])
def test_gemm_fp8_lm_head_shape(N):
    """The dense projection with E4M3 weights (the LM head of the FP8 checkpoint, 16384 rows x 2048) for 32 and
    200 token rows, against the dequantized product on sampled columns."""
    M, K = 16384, 2048
    x = synth.normal((N, K), 1.0, 11, "gfl_x", DEV)
    wq, sc = synth.fp8_rows(synth.normal((M, K), 0.02, 11, "gfl_w", DEV))
    y = torch.empty((N, M), dtype=torch.bfloat16, device=DEV)
    bd.gemm(x, wq, y, N, M, K, bd.BF16, w_scale=sc)
    torch.cuda.synchronize()
    cols = np.random.default_rng(5).choice(M, 256, replace=False)
    we = O.dequant_rows(wq[cols].cpu().numpy(), sc[cols].cpu().numpy())
    want = O.store(to64(x) @ we.T, "bf16")
    assert_close(to64(y)[:, cols], want, "bf16", "FP8 LM-head logits")


def test_gemm_fp8_every_code_exact():
    """Every E4M3 code, the subnormal ones included, reaches the tensor cores with its exact value: weight rows
    hold all 254 non-NaN codes in rotated order (scale 1), the token rows are one-hot, so every output is a single
    code's value (exact in bf16) and must equal the oracle's E4M3 definition bit for bit."""
    M, K, N = 256, 128, 128
    m, k = np.meshgrid(np.arange(M), np.arange(K), indexing="ij")
    codes = ((m + 3 * k) % 256).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0                       # the two NaN codes -> +0
    wq = torch.from_numpy(codes).to(DEV)
    sc = torch.ones(M, dtype=torch.float32, device=DEV)
    x = torch.zeros((N, K), dtype=torch.bfloat16, device=DEV)
    x[torch.arange(N), torch.arange(N) % K] = 1.0
    y = torch.empty((N, M), dtype=torch.bfloat16, device=DEV)
    bd.gemm(x, wq, y, N, M, K, bd.BF16, w_scale=sc)
    torch.cuda.synchronize()
    want = O.e4m3_value(codes).T[np.arange(N) % K]          # y[n, m] = value(code[m, n])
    assert np.array_equal(to64(y), want)


# ------------------------------------------------------------------------------------------------ attention
def _attn_case(dtype, B, Lq, Hq, Hkv, d, blk, q_pos0, n_keys, cap, key_pos=None, seed=0, nan_tail=False):
    t = _tdt(dtype)
    q = synth.normal((B, Lq, Hq, d), 1.0, seed, "aq", DEV, t)
    kc = synth.normal((B, Hkv, cap, d), 1.0, seed, "ak", DEV, t)
    vc = synth.normal((B, Hkv, cap, d), 1.0, seed, "av", DEV, t)
    if nan_tail:      # cache rows past n_keys are never read
        kc[:, :, n_keys:] = float("nan")
        vc[:, :, n_keys:] = float("nan")
    out = torch.full((B, Lq, Hq * d), float("nan"), dtype=t, device=DEV)
    kp = None if key_pos is None else torch.from_numpy(key_pos.astype(np.int32)).to(DEV)
    bd.block_attn(q, kc, vc, out, B, Lq, Hq, Hkv, d, blk, q_pos0, n_keys, cap, DT[dtype], key_pos=kp)
    torch.cuda.synchronize()
    got = to64(out).reshape(B, Lq, Hq, d)
    for b in range(B):
        kpos = np.arange(n_keys) if key_pos is None else key_pos[b]
        want = O.store(O.attention(to64(q[b]), to64(kc[b, :, :n_keys]).transpose(1, 0, 2),
                                   to64(vc[b, :, :n_keys]).transpose(1, 0, 2), np.arange(q_pos0, q_pos0 + Lq), kpos,
                                   blk), dtype)
        assert_close(got[b], want, dtype, f"attention row {b}")


def test_attention_decode_block():
    P, L = 1024, 32
    _attn_case("bf16", 1, L, 16, 4, 128, L, P, P + L, P + L)


def test_attention_decode_ragged_prefix_batch():
    P, L = 100, 32
    _attn_case("bf16", 3, L, 16, 4, 128, L, P, P + L, P + L + 5, seed=1)


def test_attention_thinned_prefix():
    P, L, n_keep, B = 300, 32, 150, 2
    g = np.random.default_rng(7)
    kp = np.stack([np.concatenate([np.sort(g.choice(P, n_keep, replace=False)), np.arange(P, P + L)])
                   for _ in range(B)])
    _attn_case("bf16", B, L, 16, 4, 128, L, P, n_keep + L, n_keep + L + 8, key_pos=kp, seed=2)


def test_attention_prefill_block_causal():
    _attn_case("bf16", 2, 96, 16, 4, 128, 32, 0, 96, 96, seed=3)


def test_attention_ragged_queries_small_blocks():
    _attn_case("bf16", 1, 70, 8, 2, 128, 16, 0, 70, 80, seed=4)


def test_attention_long_prefix_split():
    _attn_case("bf16", 2, 32, 16, 4, 128, 32, 4096, 4128, 4128, seed=5)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (16, 2), (8, 4), (32, 1)])
def test_attention_group_sizes(Hq, Hkv):
    _attn_case("bf16", 2, 32, Hq, Hkv, 128, 32, 160, 192, 200, seed=7)


def test_attention_far_positions_small_blocks():
    """Positions far past the cache rows with one-token blocks (block indices beyond 2^15)."""
    _attn_case("bf16", 1, 32, 16, 4, 128, 1, 100000, 300, 300, seed=9)
    g = np.random.default_rng(10)
    kp = np.sort(g.choice(np.arange(60000, 100000), 300, replace=False))[None, :]
    _attn_case("bf16", 1, 32, 16, 4, 128, 7, 99990, 300, 300, key_pos=kp, seed=10)


def test_attention_cache_tail_never_read():
    _attn_case("bf16", 2, 32, 16, 4, 128, 32, 200, 232, 300, seed=8, nan_tail=True)
    _attn_case("f32", 1, 16, 4, 4, 64, 16, 40, 56, 80, seed=8, nan_tail=True)


def test_attention_f32_mha():
    _attn_case("f32", 1, 16, 4, 4, 64, 16, 64, 80, 80, seed=6)


# ------------------------------------------------------------------------------------------------ SPRINT
@pytest.mark.parametrize("B,P,n_keep,cap_thin", [(2, 300, 150, 170), (1, 4096, 2048, 2080), (3, 64, 64, 64),
                                                 (1, 33, 1, 8)])
def test_prefix_retain(B, P, n_keep, cap_thin):
    Hkv, d = 4, 128
    cap = P + 16
    kc = synth.normal((B, Hkv, cap, d), 1.0, 8, "pk", DEV)
    vc = synth.normal((B, Hkv, cap, d), 1.0, 8, "pv", DEV)
    if P > 20:
        kc[:, :, 7] = kc[:, :, 3]          # exact ties: the lower position must win
        kc[:, :, 19] = kc[:, :, 3]
    keep = torch.full((B, cap_thin), -1, dtype=torch.int32, device=DEV)
    kt = torch.zeros((B, Hkv, cap_thin, d), dtype=torch.bfloat16, device=DEV)
    vt = torch.zeros_like(kt)
    sc = torch.zeros((B, P), dtype=torch.float32, device=DEV)
    bd.prefix_retain(kc, vc, keep, kt, vt, B, Hkv, d, P, cap, n_keep, cap_thin, bd.BF16, scores=sc)
    torch.cuda.synchronize()
    for b in range(B):
        o_keep, o_sc, margin = O.prefix_retain(to64(kc[b, :, :P]), None, n_keep=n_keep)
        assert len(o_keep) == n_keep
        g_keep = keep[b, :n_keep].cpu().numpy()
        assert np.allclose(to64(sc[b]), o_sc, rtol=2e-6)
        if margin > 1e-6 * np.max(o_sc):
            assert np.array_equal(g_keep, o_keep)
        assert np.all(np.diff(g_keep) > 0)
        idx = torch.from_numpy(g_keep.astype(np.int64)).to(DEV)
        assert torch.equal(kt[b, :, :n_keep], kc[b][:, idx]) and torch.equal(vt[b, :, :n_keep], vc[b][:, idx])


@pytest.mark.parametrize("B,P,n_keep,n_img,n_keep_img,alpha", [(2, 300, 150, 200, 100, 0.5), (1, 4096, 2048, 2560, 1536, 0.5),
                                                             (2, 96, 60, 40, 40, 0.0), (3, 64, 40, 50, 30, 1.0),
                                                             (1, 40, 30, 10, 20, 0.5)])
def test_prefix_retain_mixed_importance_and_modality(B, P, n_keep, n_img, n_keep_img, alpha):
    """SPRINT selection with the importance alpha l~ + (1 - alpha) c and per-modality counts (the first n_img
    positions are image tokens): kept positions against the oracle wherever each modality's selection margin is
    clear, exactly n_keep of them, n_keep_img images (or all images with the rest text when there are fewer)."""
    Hkv, d = 4, 128
    cap = P + 16
    kc = synth.normal((B, Hkv, cap, d), 1.0, 9, "pmk", DEV)
    vc = synth.normal((B, Hkv, cap, d), 1.0, 9, "pmv", DEV)
    conf = synth.uniform((B, P), 0.0, 1.0, 9, "pmc", DEV)
    mod = torch.zeros(P, dtype=torch.uint8, device=DEV)
    mod[:n_img] = 1
    keep = torch.full((B, n_keep + 4), -1, dtype=torch.int32, device=DEV)
    kt = torch.zeros((B, Hkv, n_keep + 4, d), dtype=torch.bfloat16, device=DEV)
    vt = torch.zeros_like(kt)
    sc = torch.zeros((B, P), dtype=torch.float32, device=DEV)
    bd.prefix_retain(kc, vc, keep, kt, vt, B, Hkv, d, P, cap, n_keep, n_keep + 4, bd.BF16, scores=sc, conf=conf,
                     alpha=alpha, modality=mod, n_keep_img=n_keep_img)
    torch.cuda.synchronize()
    m = mod.cpu().numpy()
    for b in range(B):
        o_keep, o_sc, margin = O.prefix_retain(to64(kc[b, :, :P]), None, n_keep=n_keep, conf=to64(conf[b]),
                                               alpha=alpha, modality=m, n_keep_img=n_keep_img)
        g_keep = keep[b, :n_keep].cpu().numpy()
        assert np.allclose(to64(sc[b]), o_sc, rtol=2e-6, atol=1e-7)
        assert len(o_keep) == n_keep and np.all(np.diff(g_keep) > 0) and g_keep.min() >= 0 and g_keep.max() < P
        assert int(m[g_keep].sum()) == int(m[o_keep].sum())
        if margin > 1e-6 * np.max(o_sc):
            assert np.array_equal(g_keep, o_keep)
        idx = torch.from_numpy(g_keep.astype(np.int64)).to(DEV)
        assert torch.equal(kt[b, :, :n_keep], kc[b][:, idx]) and torch.equal(vt[b, :, :n_keep], vc[b][:, idx])


# ------------------------------------------------------------------------------------------------ unmask
def _unmask_case(B, L, V, masked_frac, t, T_s, mode, std, cfg=0, scale=2.0, tau=0.9, k_max=8, voff=0,
                 dtype="bf16", seed=0, count_excess=None, score=0, iscale=1.0, zi_near=None):
    """cfg 0, 1 (two-way) or 2 (editing: rows per position (full, image only, unconditional)). count_excess: the
    call's row capacity is exactly the masked count n and the device count says n + count_excess; the library must
    treat it as n (the logits hold n rows per group). zi_near: with cfg 2, the image-only rows are the full rows
    plus noise of this size (close rows, as a real model's are, so that the text term cancels to a small
    difference)."""
    cfg = int(cfg)
    g = np.random.default_rng(seed)
    Btot = (1 + cfg) * B
    mask = (g.uniform(size=(B, L)) < masked_frac).astype(np.uint8)
    mask[0, 0] = 1
    mask = np.concatenate([mask] * (1 + cfg))
    tokens = np.where(mask == 1, V - 1, g.integers(0, V, (Btot, L))).astype(np.int32)
    row_pos = np.nonzero(mask[:B].reshape(-1))[0].astype(np.int32)
    n = len(row_pos)
    t_dt = _tdt(dtype)
    logits = synth.normal(((1 + cfg) * n, V), std, seed, f"ul{V}", DEV, t_dt)
    if cfg == 2 and zi_near is not None:
        noise = synth.normal((n, V), zi_near, seed, f"ul{V}_zi", DEV, torch.float32)
        logits[n:2 * n] = (logits[:n].float() + noise).to(t_dt)
    dm = torch.from_numpy(mask).to(DEV)
    dt_ = torch.from_numpy(tokens).to(DEV)
    sel = torch.empty((B, L), dtype=torch.int32, device=DEV)
    nsel = torch.empty(B, dtype=torch.int32, device=DEV)
    conf = torch.empty((B, L), dtype=torch.float32, device=DEV)
    rem = torch.empty(1, dtype=torch.int32, device=DEV)
    rp = torch.from_numpy(np.concatenate([row_pos, np.zeros(B * L - n, np.int32)])).to(DEV)
    nd = torch.tensor([n if count_excess is None else n + count_excess], dtype=torch.int32, device=DEV)
    cap = B * L if count_excess is None else n
    bd.unmask(logits, rp, nd, dt_, dm, sel, nsel, conf, rem, B, L, V, cap, t, T_s, DT[dtype], mode=mode, tau=tau,
              k_max=k_max, cfg=cfg, cfg_scale=scale, vocab_offset=voff, score=score, cfg_image_scale=iscale)
    torch.cuda.synchronize()
    zl = to64(logits)
    u = O.unmask(zl[:n], row_pos, tokens, mask, t, T_s, mode, float(np.float32(tau)), k_max, voff,
                 z_uncond=zl[cfg * n:] if cfg else None, cfg_scale=float(np.float32(scale)), score=O.SCORES[score],
                 z_image=zl[n:2 * n] if cfg == 2 else None, cfg_image_scale=float(np.float32(iscale)))
    check_unmask(u, conf.cpu().numpy(), nsel.cpu().numpy(), sel.cpu().numpy(), dt_.cpu().numpy(), dm.cpu().numpy(),
                 B, cfg)
    assert rem.item() == int(dm[:B].sum().item())
    return u


@pytest.mark.parametrize("V", [157184, 16384, 1001])
def test_unmask_fixed(V):
    _unmask_case(2, 32, V, 0.8, 1, 8, bd.FIXED, 1.0, seed=V % 97)


def test_unmask_first_step_all_masked_full_vocab():
    _unmask_case(1, 32, 157184, 1.0, 0, 8, bd.FIXED, 1.0, seed=11)


def test_unmask_threshold_crosses_tau():
    # wide logits so that some confidences exceed 0.9 and the cap of 8 binds
    u = _unmask_case(16, 32, 157184, 1.0, 0, 32, bd.THRESHOLD, 6.0, seed=12)
    assert np.any(u["nsel"] > 1)


def test_unmask_cfg_image_slice():
    _unmask_case(1, 32, 16384, 0.7, 2, 8, bd.FIXED, 1.0, cfg=True, scale=2.0, voff=157184 - 16384, seed=13)


@pytest.mark.parametrize("scale,iscale,near", [(4.0, 1.0, 0.3), (7.5, 1.5, 0.1), (4.0, 1.0, None)])
def test_unmask_editing_guidance_image_slice(scale, iscale, near):
    """Editing guidance (three rows per position) on the image-token slice: confidences, counts, chosen positions
    and the tokens written to all three row groups against the oracle, at the editing example's text scale 4.0 and
    a larger pair, with image-only rows close to the full rows and unrelated ones."""
    _unmask_case(2, 32, 16384, 0.7, 2, 8, bd.FIXED, 1.0, cfg=2, scale=scale, iscale=iscale,
                 voff=157184 - 16384, seed=17, zi_near=near)


@pytest.mark.parametrize("score", [0, 1, 2], ids=["low_confidence", "top_k_margin", "neg_entropy"])
def test_unmask_editing_guidance_scores_full_vocab(score):
    """Editing guidance through each ranking's reduction (the largest-probability one and the extended one of the
    other scores) over the full vocabulary, whose 157184 entries are not a multiple of the vector chunk, with
    threshold acceptance; fp32 logits check the scalar tail of the same kernels."""
    _unmask_case(1, 32, 157184, 1.0, 1, 8, 1, 3.0, cfg=2, scale=4.0, iscale=1.25, seed=50 + score, score=score,
                 zi_near=0.5)
    _unmask_case(2, 16, 1001, 0.8, 0, 4, bd.FIXED, 1.0, cfg=2, scale=2.0, iscale=0.5, seed=53 + score, score=score,
                 dtype="f32")


def test_unmask_last_step_takes_all():
    u = _unmask_case(3, 32, 4096, 0.3, 7, 8, bd.FIXED, 1.0, seed=14)
    assert np.all(u["mask"] == 0)


def test_unmask_f32():
    _unmask_case(1, 16, 1024, 1.0, 0, 4, bd.FIXED, 1.0, dtype="f32", seed=15)


@pytest.mark.parametrize("score", [1, 2], ids=["top_k_margin", "neg_entropy"])
@pytest.mark.parametrize("mode", [0, 1], ids=["fixed", "threshold"])
def test_unmask_position_scores(score, mode):
    """The other ranking strategies (top-2 margin, negated entropy): confidences (largest probability), counts,
    chosen positions in rank order and written tokens against the oracle, on rows whose logits spread widely enough
    that the threshold and the ranking both matter."""
    _unmask_case(4, 32, 16384, 0.9, 0, 8, mode, 4.0, seed=40 + score + 2 * mode, score=score)


@pytest.mark.parametrize("score", [1, 2], ids=["top_k_margin", "neg_entropy"])
def test_unmask_position_scores_cfg_full_vocab(score):
    _unmask_case(1, 32, 157184, 1.0, 1, 8, 1, 3.0, cfg=True, scale=2.0, seed=45 + score, score=score)


@pytest.mark.parametrize("cfg", [0, 1, 2])
def test_unmask_device_count_above_capacity_is_clamped(cfg):
    """A device row count above the call's max_rows is read as max_rows: no partial or logit row beyond the
    capacity is touched, and the result is that of the true count."""
    _unmask_case(3, 32, 16384, 0.6, 1, 8, bd.FIXED, 1.0, cfg=cfg, seed=16, count_excess=9)


# ------------------------------------------------------------------------------------------------ failure path
def test_bounded_wait_reports_timeout_and_recovers():
    """A wait that can never complete gives up after its bound, the status word says so, the context stays usable."""
    lib = bd.load()
    ws = bd.Workspace(4096, DEV)
    assert bd.status_check(ws) == bd.OK
    bd.check(lib.dllm_selftest_bounded_wait(ws.addr, ws.nbytes, bd.stream_handle()))
    assert bd.status_check(ws) == bd.ERR_TIMEOUT
    assert bd.status_check(ws) == bd.OK                      # the check clears the word
    x = torch.ones(8, device=DEV)                            # the context still works
    assert float((x * 2).sum().item()) == 16.0
