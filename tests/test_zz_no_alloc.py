"""dllm_unmask_noalloc against dllm_unmask (GPU).

The allocation-free variant serves callers that cannot allocate device memory (a plug-in whose host owns the
device memory pool, a serving loop that forbids cudaMalloc after start-up). It keeps its scratch in a fixed array
inside the library instead of a caller workspace. Here both entry points get the same inputs through the C ABI,
twice in a row (the second call finds the first call's leftovers in the shared array), and must agree exactly on
the integer results and within the confidence tolerance of the other unmask tests. This file is collected last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from block_diffusion_moe_dllm_b200 import binding as bd
from block_diffusion_moe_dllm_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(B, L, V, seed, cfg):
    g = np.random.default_rng(seed)
    mask = (g.uniform(size=(B, L)) < 0.75).astype(np.uint8)
    mask[:, 0] = 1
    mask = np.concatenate([mask] * (1 + cfg))   # every guidance row group shares the pattern
    tokens = np.where(mask == 1, V - 1, g.integers(0, V, mask.shape)).astype(np.int32)
    row_pos = np.nonzero(mask[:B].reshape(-1))[0].astype(np.int32)
    n = len(row_pos)
    logits = synth.normal(((1 + cfg) * n, V), 3.0, seed, f"noalloc{V}", DEV)
    rp = torch.from_numpy(np.concatenate([row_pos, np.zeros(B * L - n, np.int32)])).to(DEV)
    nd = torch.tensor([n], dtype=torch.int32, device=DEV)
    return logits, rp, nd, torch.from_numpy(tokens).to(DEV), torch.from_numpy(mask).to(DEV)


def _outputs(B, L):
    return (torch.full((B, L), -7, dtype=torch.int32, device=DEV), torch.full((B,), -7, dtype=torch.int32, device=DEV),
            torch.full((B, L), -7.0, dtype=torch.float32, device=DEV), torch.full((1,), -7, dtype=torch.int32, device=DEV))


@pytest.mark.parametrize("B,L,V,t,T_s,mode,cfg", [(16, 32, 157184, 0, 32, bd.THRESHOLD, 0),
                                                  (2, 32, 16384, 1, 8, bd.FIXED, 1),
                                                  (2, 32, 16384, 1, 8, bd.FIXED, 2)])
def test_unmask_noalloc_matches_workspace_version(B, L, V, t, T_s, mode, cfg):
    lib = bd.load()
    desc = bd.UnmaskDesc(B, L, V, B * L, t, T_s, mode, 0.9, 8, cfg, 2.0, 0, bd.BF16, 0, 1.5)
    need = lib.dllm_unmask_workspace_size(C.byref(desc))
    ws = bd.Workspace(need, DEV)
    stream = bd.stream_handle()
    for call in range(2):
        logits, rp, nd, tok, msk = _inputs(B, L, V, seed=100 + call, cfg=cfg)
        tok_a, msk_a = tok.clone(), msk.clone()
        tok_b, msk_b = tok.clone(), msk.clone()
        sel_a, nsel_a, conf_a, rem_a = _outputs(B, L)
        sel_b, nsel_b, conf_b, rem_b = _outputs(B, L)
        bd.check(lib.dllm_unmask(C.byref(desc), bd.ptr(logits), bd.ptr(rp), bd.ptr(nd), bd.ptr(tok_a), bd.ptr(msk_a),
                                 bd.ptr(sel_a), bd.ptr(nsel_a), bd.ptr(conf_a), bd.ptr(rem_a), ws.addr, ws.nbytes,
                                 stream))
        bd.check(lib.dllm_unmask_noalloc(C.byref(desc), bd.ptr(logits), bd.ptr(rp), bd.ptr(nd), bd.ptr(tok_b),
                                         bd.ptr(msk_b), bd.ptr(sel_b), bd.ptr(nsel_b), bd.ptr(conf_b), bd.ptr(rem_b),
                                         stream))
        torch.cuda.synchronize()
        assert torch.equal(tok_a, tok_b) and torch.equal(msk_a, msk_b), f"call {call}: tokens/mask differ"
        assert torch.equal(sel_a, sel_b) and torch.equal(nsel_a, nsel_b) and torch.equal(rem_a, rem_b)
        ca, cb = conf_a.double().cpu().numpy(), conf_b.double().cpu().numpy()
        assert np.all(np.abs(ca - cb) <= 1e-6 * np.maximum(np.abs(ca), 1e-30) + 1e-12), f"call {call}: confidences"
        assert int(nsel_b.sum().item()) > 0


def test_unmask_noalloc_rejects_oversized_request():
    lib = bd.load()
    # 32768 masked rows x at least ceil(157184 / 32768) = 5 vocabulary chunks x 16 bytes = 2.5 MiB of partials,
    # far above the fixed 256 KiB: rejected on the host before any launch (the buffers below are never touched)
    desc = bd.UnmaskDesc(1024, 32, 157184, 1024 * 32, 0, 8, bd.FIXED, 0.9, 8, 0, 1.0, 0, bd.BF16)
    z = torch.zeros(16, dtype=torch.int32, device=DEV)
    rc = lib.dllm_unmask_noalloc(C.byref(desc), bd.ptr(z), bd.ptr(z), bd.ptr(z), bd.ptr(z), bd.ptr(z), bd.ptr(z),
                                 bd.ptr(z), bd.ptr(z), bd.ptr(z), bd.stream_handle())
    assert rc == bd.ERR_UNSUPPORTED
    assert "scratch" in lib.dllm_last_error().decode()


def test_unmask_noalloc_limit_is_exactly_16384_partials():
    """With a 16384-entry vocabulary and thousands of rows every row is one chunk, so the partials needed equal
    max_rows: 16384 rows (256 KiB, the whole array) are accepted and agree with dllm_unmask; 16385 are rejected."""
    lib = bd.load()
    B, L, V = 512, 32, 16384
    desc = bd.UnmaskDesc(B, L, V, B * L, 1, 8, bd.FIXED, 0.9, 8, 0, 1.0, 0, bd.BF16)
    # a quarter of the positions masked keeps the logits at 128 MB; the capacity is still 16384 rows
    g = np.random.default_rng(7)
    mask = (g.uniform(size=(B, L)) < 0.25).astype(np.uint8)
    mask[:, 0] = 1
    tokens = np.where(mask == 1, V - 1, g.integers(0, V, mask.shape)).astype(np.int32)
    row_pos = np.nonzero(mask.reshape(-1))[0].astype(np.int32)
    n = len(row_pos)
    logits = synth.normal((n, V), 3.0, 7, "noalloc-limit", DEV)
    rp = torch.from_numpy(np.concatenate([row_pos, np.zeros(B * L - n, np.int32)])).to(DEV)
    nd = torch.tensor([n], dtype=torch.int32, device=DEV)
    need = lib.dllm_unmask_workspace_size(C.byref(desc))
    ws = bd.Workspace(need, DEV)
    stream = bd.stream_handle()
    res = []
    for noalloc in (False, True):
        tok, msk = torch.from_numpy(tokens).to(DEV), torch.from_numpy(mask).to(DEV)
        sel, nsel, conf, rem = _outputs(B, L)
        args = [bd.ptr(logits), bd.ptr(rp), bd.ptr(nd), bd.ptr(tok), bd.ptr(msk), bd.ptr(sel), bd.ptr(nsel),
                bd.ptr(conf), bd.ptr(rem)]
        if noalloc:
            bd.check(lib.dllm_unmask_noalloc(C.byref(desc), *args, stream))
        else:
            bd.check(lib.dllm_unmask(C.byref(desc), *args, ws.addr, ws.nbytes, stream))
        res.append((tok, msk, sel, nsel, conf, rem))
    torch.cuda.synchronize()
    a, b = res
    for i in (0, 1, 2, 3, 5):
        assert torch.equal(a[i], b[i])
    ca, cb = a[4].double().cpu().numpy(), b[4].double().cpu().numpy()
    assert np.all(np.abs(ca - cb) <= 1e-6 * np.maximum(np.abs(ca), 1e-30) + 1e-12)
    # one row more than the array holds: rejected before any launch
    over = bd.UnmaskDesc(B + 1, L, V, B * L + 1, 1, 8, bd.FIXED, 0.9, 8, 0, 1.0, 0, bd.BF16)
    z = torch.zeros(16, dtype=torch.int32, device=DEV)
    rc = lib.dllm_unmask_noalloc(C.byref(over), bd.ptr(z), bd.ptr(z), bd.ptr(z), bd.ptr(z), bd.ptr(z), bd.ptr(z),
                                 bd.ptr(z), bd.ptr(z), bd.ptr(z), stream)
    assert rc == bd.ERR_UNSUPPORTED
