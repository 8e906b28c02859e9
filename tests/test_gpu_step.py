"""End-to-end parity of dllm_denoise_step (the whole pass through the C ABI) against the fp64 oracle (GPU).

Both sides start from the same seeded weights, caches and block state. The oracle never sees a value the
library computed. Where the two may legitimately part (a routing or confidence near-tie that a rounding
difference can flip), the affected rows are excluded and counted, and a block comparison stops at the first
such step.
"""
import numpy as np
import pytest
import torch

from block_diffusion_moe_dllm_b200 import binding as bd
from block_diffusion_moe_dllm_b200 import synth
from block_diffusion_moe_dllm_b200.configs import ONE_LAYER, TINY_F32, scaled
from block_diffusion_moe_dllm_b200.engine import DenoiseEngine
from oracle import dllm_oracle as O
from _util import assert_close, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"

# small bf16 backbone with the tensor-core path's constraints (head dim 128, H % 128 == 0, I % 64 == 0)
SMALL = scaled(ONE_LAYER, name="small-bf16", n_layers=2, H=256, Hq=2, Hkv=1, d=128, E=8, k=2, I=128, V=1024, B=2,
               P=64, L=16, T_s=4)
# Routing margins below this can flip when the two sides' bf16 router inputs differ by one ulp in a few
# elements: one ulp (2^-7 relative, ~8e-3 at |h| ~ 1) times a router weight (~0.02) moves a logit by ~1.6e-4
# and a sigmoid score by at most a quarter of that; 3e-4 leaves a margin for a handful of such elements at hidden
# size 256. The elements whose rounding differs add up like a random walk, so the band grows as sqrt(H / 256).
# fp32 storage: 1e-5.
E2E_ROUTE_MARGIN = 3e-4
E2E_CONF_MARGIN = 2e-2    # relative confidence margins below this can flip under one-ulp logit differences


def _setup(w, seed=0, masked_fraction=1.0, random_gains=True):
    wt = synth.make_weights(w, DEV, seed=seed, random_gains=random_gains)
    caches = synth.make_prefix_cache(w, DEV, seed=seed)
    tokens, mask = synth.make_block_state(w, DEV, seed=seed, masked_fraction=masked_fraction)
    eng = DenoiseEngine(w, wt, caches, DEV)
    eng.set_block(tokens, mask)
    return wt, caches, eng, tokens.cpu().numpy(), mask.cpu().numpy()


def _host(wt):
    """Host copies of the weights for the oracle (the same bytes the library reads); FP8 matrices (codes with a
    "<name>_scale" entry) are handed over as their dequantized values (the oracle's E4M3 definition, exact)."""
    cp = lambda t: t.detach().cpu()

    def conv(d, name):
        if name + "_scale" in d:
            return O.dequant_rows(cp(d[name]).numpy(), cp(d[name + "_scale"]).numpy())
        return cp(d[name])
    return {"embed": cp(wt["embed"]), "final_norm": cp(wt["final_norm"]), "w_lm": conv(wt, "w_lm"),
            "layers": [{k: conv(lw, k) for k in lw if not k.endswith("_scale")} for lw in wt["layers"]]}


def _host_caches(caches, P):
    return [(c[0][:, :, :P].cpu(), c[1][:, :, :P].cpu()) for c in caches]


def _route_margin(dtype, H=256):
    return E2E_ROUTE_MARGIN * max(1.0, (H / 256) ** 0.5) if dtype == "bf16" else 1e-5


def _flagged_tokens(f, dtype="bf16", H=256):
    flag = np.zeros(f["x"].shape[0] * f["x"].shape[1], dtype=bool)
    for r in f["route"]:
        if r is not None:
            flag |= r[2] < _route_margin(dtype, H)
    return flag


def _check_pass(w, eng, f, dtype):
    n = len(f["row_pos"])
    flag = _flagged_tokens(f, dtype, w.H)
    x = to64(eng.x_final()).reshape(w.B * w.L, w.H)
    ok = ~flag
    assert ok.sum() >= 0.5 * len(ok), "too many routing near-ties for a meaningful comparison"
    assert_close(x[ok], f["x"].reshape(-1, w.H)[ok], dtype, "hidden state after the last layer", ulps=2)
    lg = to64(eng.logits(n))
    groups = 1 + w.cfg
    Bl = w.B // groups
    rows = [p + g * Bl * w.L for g in range(groups) for p in f["row_pos"]]
    okr = ~flag[np.asarray(rows, dtype=np.int64)]
    if w.cfg:  # a guided row needs all of its rows clean
        okr = np.tile(okr.reshape(groups, n).all(axis=0), groups)
    assert_close(lg[okr], f["logits"][okr], dtype, "logits of the masked rows", ulps=2,
                 scale=max(1.0, w.lm_std / 0.02))
    return flag


def _score_shift(score, r, c, dz):
    """First-order bound on how far a position score r (largest probability c) moves when every logit of the row
    moves by at most dz: dp_v = p_v (dz_v - sum_u p_u dz_u), so |dp_v| <= 2 dz p_v. top_k_margin p1 - p2 moves by
    at most 2 dz (p1 + p2) <= 4 dz c; neg_entropy sum_v p_v log p_v moves by sum_v |log p_v + 1| |dp_v|
    <= 2 dz (|r| + 1)."""
    if score == 1:
        return 4.0 * dz * c
    return 2.0 * dz * (abs(r) + 1.0)


def _guidance_gain(w):
    """How much guidance can scale a common difference dz of its rows' logits: z = zu + s (zc - zu) moves by at
    most (|1 - s| + |s|) dz; z = zu (1 - s_i) + zi (s_i - s_t) + zc s_t by at most (|1 - s_i| + |s_i - s_t| +
    |s_t|) dz."""
    if w.cfg == 2:
        return abs(1.0 - w.cfg_image_scale) + abs(w.cfg_image_scale - w.cfg_scale) + abs(w.cfg_scale)
    if w.cfg:
        return abs(1.0 - w.cfg_scale) + abs(w.cfg_scale)
    return 1.0


def _decisions_agree(w, u_or, eng, flag):
    """Compare the unmask decisions where the oracle's choice is not a near-tie (ranking by the workload's score,
    threshold on the largest probability). For the margin and entropy scores the near-tie band also covers what
    the observed difference between the two sides' logits (dz, largest over the scored rows, scaled by the
    guidance) can move the scores by."""
    Bl = w.B // (1 + w.cfg)
    dz = 0.0
    if w.score:
        f = u_or["forward"]
        n = len(f["row_pos"])
        dz = float(np.max(np.abs(to64(eng.logits(n)) - f["logits"]))) if n else 0.0
        dz *= _guidance_gain(w)
    g_mask = eng.mask.cpu().numpy()
    g_nsel = eng.nsel.cpu().numpy()
    clean = True
    for b in range(Bl):
        c = u_or["conf"][b]
        rk = u_or["rank"][b][c > 0]
        row_flag = any(flag[(b + g * Bl) * w.L:(b + g * Bl + 1) * w.L].any() for g in range(1 + w.cfg))
        order = np.argsort(-rk, kind="stable")
        ranked, c_ranked = rk[order], c[c > 0][order]
        k = u_or["nsel"][b]
        near = False
        if 0 < k < len(ranked):
            gap = ranked[k - 1] - ranked[k]
            near = gap < E2E_CONF_MARGIN * max(abs(ranked[k - 1]), 1e-30)
            if w.score:   # the band a logit difference of up to dz can move the two scores by
                near |= gap < 2.0 * (_score_shift(w.score, ranked[k - 1], c_ranked[k - 1], dz) +
                                     _score_shift(w.score, ranked[k], c_ranked[k], dz))
        if w.mode == 1:
            near |= bool(np.any(np.abs(c[c > 0] - w.tau) < E2E_CONF_MARGIN))
        if near or row_flag:
            clean = False
            continue
        assert g_nsel[b] == u_or["nsel"][b]
        assert np.array_equal(g_mask[b], u_or["mask"][b]), f"row {b}: unmasked positions differ"
    return clean


def _check_candidates(w, eng, u_or, f, flag):
    """Candidate tokens written this step agree wherever the oracle's top-2 logit gap is clear."""
    n = len(f["row_pos"])
    z = f["logits"][:n]
    if w.cfg == 2:
        z = O.cfg3_combine(z, f["logits"][n:2 * n], f["logits"][2 * n:], w.cfg_scale, w.cfg_image_scale)
    elif w.cfg:
        z = O.cfg_combine(z, f["logits"][n:], w.cfg_scale)
    top2 = np.sort(z, axis=1)[:, -2:]
    clear = (top2[:, 1] - top2[:, 0]) > 0.05
    g_tok = eng.tokens.cpu().numpy()
    g_mask = eng.mask.cpu().numpy()
    for r, p in enumerate(f["row_pos"]):
        b, i = divmod(int(p), w.L)
        if not clear[r] or flag[p] or g_mask[b, i] == 1 or u_or["mask"][b, i] == 1:
            continue
        assert g_tok[b, i] == u_or["cand"][b, i], f"candidate token at row {b} pos {i}"


def _one_pass(w, seed=0, masked_fraction=1.0, t=0, random_gains=True):
    wt, caches, eng, tok0, mask0 = _setup(w, seed, masked_fraction, random_gains)
    hw, hc = _host(wt), _host_caches(caches, w.P)
    keep = None
    if w.sprint:
        conf = eng.prefix_conf.cpu().numpy() if eng.prefix_conf is not None else None
        mod = eng.prefix_modality.cpu().numpy() if eng.prefix_modality is not None else None
        keep = O.sprint_keep(w, hc, conf=conf, modality=mod)
    eng.step(t)
    torch.cuda.synchronize()
    assert bd.status_check(eng.ws) == bd.OK
    u = O.denoise_step(w, hw, hc, tok0, mask0, t, keep=keep)
    flag = _check_pass(w, eng, u["forward"], w.dtype)
    _decisions_agree(w, u, eng, flag)
    _check_candidates(w, eng, u, u["forward"], flag)
    if w.sprint:
        for l in range(w.n_layers):
            kp = eng.thin[l][2]
            for b in range(w.B):
                got = kp[b, : w.n_keep].cpu().numpy()
                _, sc, margin = O.prefix_retain(O.f64(hc[l][0][b]), None, n_keep=w.n_keep,
                                                conf=None if conf is None else conf[b][: w.P], alpha=w.sprint_alpha,
                                                modality=None if mod is None else mod[: w.P],
                                                n_keep_img=w.n_keep_img)
                if margin > 1e-6 * sc.max():
                    assert np.array_equal(got, keep[l][b])
                assert np.array_equal(kp[b, w.n_keep: w.n_keep + w.L].cpu().numpy(), np.arange(w.P, w.P + w.L))
    return eng, u


def test_step_tiny_fp32():
    _one_pass(TINY_F32, seed=0)


def test_step_small_bf16_all_masked():
    _one_pass(SMALL, seed=1)


def test_step_small_bf16_partly_masked_mid_block():
    _one_pass(SMALL, seed=2, masked_fraction=0.5, t=2)


def test_step_small_bf16_cfg_image_slice():
    w = scaled(SMALL, B=2, cfg=1, cfg_scale=2.0, vocab_offset=1024 - 256, vocab_len=256)
    _one_pass(w, seed=3)


def test_step_small_bf16_editing_guidance():
    """Editing guidance: three rows per position (instruction and image, image only, unconditional), the
    image-token slice of the head, text scale 4 and image scale 1.5; the chosen tokens land in all three groups."""
    w = scaled(SMALL, name="small-bf16-edit", B=3, cfg=2, cfg_scale=4.0, cfg_image_scale=1.5,
               vocab_offset=1024 - 256, vocab_len=256)
    eng, u = _one_pass(w, seed=10)
    g_tok, g_mask = eng.tokens.cpu().numpy(), eng.mask.cpu().numpy()
    assert np.array_equal(g_mask[0], g_mask[1]) and np.array_equal(g_mask[0], g_mask[2])
    assert np.array_equal(g_tok[0], g_tok[1]) and np.array_equal(g_tok[0], g_tok[2])
    assert int(eng.nsel[0].item()) > 0


def test_step_small_bf16_editing_guidance_threshold():
    """Editing guidance with threshold acceptance on logits spread wide enough that confidences cross tau and the
    cap binds: counts, chosen positions and tokens of all three groups against the oracle."""
    w = scaled(SMALL, name="small-bf16-edit-thr", B=3, cfg=2, cfg_scale=4.0, cfg_image_scale=1.25, mode=1, tau=0.9,
               k_max=8, T_s=16, lm_std=1.0)
    eng, u = _one_pass(w, seed=11)
    g_mask = eng.mask.cpu().numpy()
    assert np.array_equal(g_mask[0], g_mask[1]) and np.array_equal(g_mask[0], g_mask[2])


def test_step_small_bf16_sprint():
    w = scaled(SMALL, B=3, P=96, sprint=1, keep_ratio=0.5)
    _one_pass(w, seed=4)


@pytest.mark.parametrize("score", [1, 2], ids=["top_k_margin", "neg_entropy"])
def test_step_small_bf16_position_scores(score):
    _one_pass(scaled(SMALL, name=f"small-bf16-score{score}", mode=1, tau=0.9, k_max=8, T_s=16, lm_std=1.0,
                     score=score), seed=6 + score)


def test_step_small_bf16_sprint_mixed_modality():
    """SPRINT with the mixed importance (alpha 0.5, prompt confidences 1) and modality counts: the first 64 of 96
    prefix positions are image tokens, half of them kept, all text kept."""
    w = scaled(SMALL, name="small-bf16-sprint-mixed", B=3, P=96, sprint=1, keep_ratio=1.0, sprint_alpha=0.5,
               n_img_prefix=64, img_keep_ratio=0.5)
    eng, _ = _one_pass(w, seed=9)
    assert w.n_keep == 32 + 32
    for l in range(w.n_layers):
        kp = eng.thin[l][2][:, : w.n_keep].cpu().numpy()
        assert np.all((kp < 64).sum(axis=1) == 32)


def test_step_block_rows_full_width_projections():
    """Sixteen rows of a 32-token block (512 token rows) through full-width projections (hidden 2048, 16 q heads,
    4 kv heads): the QKV projection with RoPE and cache writes and the output projection with the residual run as
    wide split-K clusters, whose ranks each write their share of the columns."""
    w = scaled(ONE_LAYER, name="block-rows-h2048", n_layers=1, E=8, k=2, I=128, V=1024, B=16, P=64, L=32, T_s=4)
    _one_pass(w, seed=13)


def test_step_small_bf16_threshold():
    w = scaled(SMALL, mode=1, tau=0.9, k_max=8, T_s=16, lm_std=1.0)
    _one_pass(w, seed=5)


# ------------------------------------------------------------------------------------------------ FP8 weights
# The expert and LM-head weights as E4M3 codes with per-row scales (the FP8 checkpoint); the oracle runs the same
# pass on the codes' exact values.

def test_step_small_fp8_weights():
    _one_pass(scaled(SMALL, name="small-fp8", wfmt="fp8"), seed=51)


def test_step_small_fp8_weights_cfg_threshold():
    w = scaled(SMALL, name="small-fp8-cfg", wfmt="fp8", B=2, cfg=1, cfg_scale=2.0, vocab_offset=1024 - 256,
               vocab_len=256)
    _one_pass(w, seed=52)


def test_step_fp8_fused_confidence():
    _one_pass(scaled(SMALL, name="small-fp8-fused", B=1, L=32, V=20480, wfmt="fp8"), seed=53, masked_fraction=0.6,
              t=2)


def test_step_fp8_cta_rows():
    """512 token rows with 16 q / 4 kv heads through FP8 experts (N tiles of 64 and 128 rows: groups of ~60 rows)."""
    _one_pass(scaled(SMALL, name="small-fp8-rows", wfmt="fp8", B=16, Hq=16, Hkv=4, P=64, L=32), seed=54)


# One logical row of at most 32 positions, no guidance, and a scored vocabulary of at least 74 weight tiles of 128
# rows: the LM head writes the confidence partials from its epilogue (one per persistent CTA) and the step launches
# no separate reduction.
FUSED = scaled(SMALL, name="small-bf16-fused-confidence", B=1, L=32, V=20480)


def test_step_fused_confidence_partly_masked():
    _one_pass(FUSED, seed=21, masked_fraction=0.6, t=2)


def test_step_fused_confidence_vocab_slice_threshold():
    w = scaled(FUSED, vocab_offset=4096, vocab_len=128 * 80, mode=1, tau=0.9, k_max=8, T_s=16, lm_std=1.0)
    _one_pass(w, seed=22)


@pytest.mark.parametrize("masked_fraction", [1.0, 0.3])
def test_fused_confidence_equals_reduction(masked_fraction):
    """The fused confidence of a step equals the standalone reduction over the logits that step wrote. The
    standalone reduction is itself held to the oracle within 1e-6 relative (the unmask tests), so this pins the
    fused epilogue and the many-partial merge of the selection to the same arithmetic."""
    w = scaled(FUSED, lm_std=0.5)
    _, _, eng, tok0, mask0 = _setup(w, seed=23, masked_fraction=masked_fraction)
    t = 1
    eng.step(t)
    torch.cuda.synchronize()
    assert bd.status_check(eng.ws) == bd.OK
    row_pos = np.nonzero(mask0.reshape(-1))[0].astype(np.int32)
    n = len(row_pos)
    logits = eng.logits(n).clone()
    dm = torch.from_numpy(mask0).to(DEV)
    dt_ = torch.from_numpy(tok0).to(DEV)
    sel = torch.empty((1, w.L), dtype=torch.int32, device=DEV)
    nsel = torch.empty(1, dtype=torch.int32, device=DEV)
    conf = torch.empty((1, w.L), dtype=torch.float32, device=DEV)
    rem = torch.empty(1, dtype=torch.int32, device=DEV)
    rp = torch.from_numpy(np.concatenate([row_pos, np.zeros(w.L - n, np.int32)])).to(DEV)
    nd = torch.tensor([n], dtype=torch.int32, device=DEV)
    bd.unmask(logits, rp, nd, dt_, dm, sel, nsel, conf, rem, 1, w.L, w.vlen, w.L, t, w.T_s, bd.BF16, mode=w.mode,
              tau=w.tau, k_max=w.k_max)
    torch.cuda.synchronize()
    m_ = mask0[0].astype(bool)
    c_step = eng.conf.cpu().numpy()[0].astype(np.float64)
    c_red = conf.cpu().numpy()[0].astype(np.float64)
    assert np.all(np.abs(c_step[m_] - c_red[m_]) <= 2e-6 * c_red[m_])
    cs = np.sort(c_red[m_])[::-1]
    k = int(nsel.item())
    if not (0 < k < len(cs) and cs[k - 1] - cs[k] < 1e-5 * cs[k - 1]):
        assert int(eng.nsel[0].item()) == k
        assert np.array_equal(eng.mask.cpu().numpy(), dm.cpu().numpy())
        assert np.array_equal(eng.tokens.cpu().numpy(), dt_.cpu().numpy())


def test_step_cta_pairs():
    """1024 tokens through 16 q / 4 kv heads: the QKV projection (24 weight tiles x 4 token tiles) and both expert
    GEMMs (~256 rows per expert) run as CTA pairs sharing each MMA, through the RoPE/cache, SwiGLU and fp32 epilogues."""
    w = scaled(SMALL, name="small-bf16-pairs", B=32, Hq=16, Hkv=4, P=64, L=32)
    _one_pass(w, seed=31)


def test_step_one_layer_full_size():
    """The one-layer bf16 workload at its full size (hidden 2048, 256 experts, vocab 157184, prefix 1024)."""
    _one_pass(ONE_LAYER, seed=0, random_gains=False)


@pytest.mark.parametrize("w", [TINY_F32, SMALL], ids=["tiny-f32", "small-bf16"])
def test_block_decode(w):
    """All T_s passes of a block. The oracle follows its own decisions from the same start; the two states are
    compared after every step until a step whose decision is a near-tie (after which they may part)."""
    wt, caches, eng, tok, mask = _setup(w, seed=7)
    hw, hc = _host(wt), _host_caches(caches, w.P)
    compared = 0
    for t in range(w.T_s):
        eng.step(t)
        torch.cuda.synchronize()
        if tok is None:
            continue
        u = O.denoise_step(w, hw, hc, tok, mask, t)
        flag = _flagged_tokens(u["forward"], w.dtype, w.H)
        clean = _decisions_agree(w, u, eng, flag)
        _check_candidates(w, eng, u, u["forward"], flag)
        if not np.array_equal(eng.mask.cpu().numpy(), u["mask"]):
            assert not clean, f"step {t}: unmasked positions differ without a near-tie"
            tok = None
            continue
        if not np.array_equal(eng.tokens.cpu().numpy(), u["tokens"]):
            tok = None          # a candidate with an unclear top-2 gap was written (checked where clear)
            continue
        compared += 1
        tok, mask = u["tokens"], u["mask"]
    assert int(eng.mask.sum().item()) == 0, "every position is unmasked after the last step"


@pytest.mark.parametrize("w", [TINY_F32, SMALL, scaled(SMALL, sprint=1, keep_ratio=0.5)],
                         ids=["tiny-f32", "small-bf16", "small-bf16-sprint"])
def test_commit_pass(w):
    """The commit pass over a seeded clean block writes each layer's block K/V into cache rows [P, P + L)."""
    wt, caches, eng, _, _ = _setup(w, seed=8)
    hw, hc = _host(wt), _host_caches(caches, w.P)
    clean = synth.randint((w.B, w.L), 0, w.V - 1, 8, "clean_block", DEV)
    eng.set_block(clean, torch.zeros((w.B, w.L), dtype=torch.uint8, device=DEV))
    keep = None
    if w.sprint:
        eng.step(0)          # selects the kept prefix (retain) for this block
        keep = O.sprint_keep(w, hc)
        eng.set_block(clean, torch.zeros((w.B, w.L), dtype=torch.uint8, device=DEV))
    eng.commit()
    torch.cuda.synchronize()
    assert bd.status_check(eng.ws) == bd.OK
    bk, bv = O.commit_block(w, hw, hc, clean.cpu().numpy(), keep=keep)
    flag = np.zeros(w.B * w.L, dtype=bool)
    f = O.forward_block(w, hw, hc, clean.cpu().numpy(), np.zeros((w.B, w.L), np.int64), keep=keep,
                        want_logits=False, skip_last_ffn=True)
    for l in range(w.n_layers):
        kc, vc = caches[l]
        got_k = to64(kc[:, :, w.P: w.P + w.L]).transpose(0, 2, 1, 3)
        got_v = to64(vc[:, :, w.P: w.P + w.L]).transpose(0, 2, 1, 3)
        ok = ~flag.reshape(w.B, w.L)
        assert_close(got_k[ok], bk[l][ok], w.dtype, f"committed K layer {l}")
        assert_close(got_v[ok], bv[l][ok], w.dtype, f"committed V layer {l}")
        # routing near-ties in this layer can change the next layer's input: mark those tokens
        if f["route"][l] is not None:
            flag |= f["route"][l][2] < _route_margin(w.dtype, w.H)


# ------------------------------------------------------------------------------------------------ early finish
def _snapshot(eng, caches):
    return (eng.tokens.clone(), eng.mask.clone(), [(k.clone(), v.clone()) for k, v in caches])


def test_block_finished_early_later_passes_do_nothing():
    """Threshold mode with tau = 0 and k_max >= L accepts every position at the first pass ([R] "SPRINT":
    accept every c > tau). The block is then finished: the remaining passes of the block launch, see no masked
    position and change nothing (tokens, mask, every layer's K/V cache); the commit pass still runs."""
    w = scaled(SMALL, name="small-bf16-early", mode=1, tau=0.0, k_max=32, T_s=6)
    wt, caches, eng, tok0, mask0 = _setup(w, seed=41)
    hw, hc = _host(wt), _host_caches(caches, w.P)
    eng.step(0)
    torch.cuda.synchronize()
    assert bd.status_check(eng.ws) == bd.OK
    u = O.denoise_step(w, hw, hc, tok0, mask0, 0)
    assert int(eng.remaining.item()) == 0 and int(eng.mask.sum().item()) == 0
    assert np.array_equal(eng.nsel.cpu().numpy(), u["nsel"]) and np.all(u["nsel"] == w.L)
    snap = _snapshot(eng, caches)
    for t in range(1, w.T_s):
        eng.step(t)
    torch.cuda.synchronize()
    assert bd.status_check(eng.ws) == bd.OK
    assert torch.equal(eng.tokens, snap[0]) and torch.equal(eng.mask, snap[1])
    for (k, v), (k0, v0) in zip(caches, snap[2]):
        assert torch.equal(k, k0) and torch.equal(v, v0), "a finished block's pass wrote the cache"
    assert int(eng.remaining.item()) == 0 and int(eng.nsel.sum().item()) == 0
    eng.commit()
    torch.cuda.synchronize()
    assert bd.status_check(eng.ws) == bd.OK
    assert not torch.equal(caches[0][0][:, :, w.P: w.P + w.L], snap[2][0][0][:, :, w.P: w.P + w.L])


def test_finished_pass_costs_only_its_launches():
    """At the one-layer workload's full size a pass over a finished block (every kernel returns at entry) takes
    a fraction of a live pass (which streams about 1 GB of weights)."""
    w = ONE_LAYER
    wt, caches, eng, _, _ = _setup(w, seed=3, random_gains=False)
    tokens, mask = synth.make_block_state(w, DEV, seed=3)
    done = torch.zeros_like(mask)

    def timed(m):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ts = []
        for _ in range(6):
            eng.set_block(tokens, m)
            torch.cuda.synchronize()
            ev[0].record()
            eng.step(1)
            ev[1].record()
            torch.cuda.synchronize()
            ts.append(ev[0].elapsed_time(ev[1]))
        return sorted(ts[1:])[2]

    live, dead = timed(mask), timed(done)
    assert bd.status_check(eng.ws) == bd.OK
    assert dead < 0.5 * live, f"finished pass {dead * 1e3:.0f} us vs live pass {live * 1e3:.0f} us"


@pytest.mark.parametrize("early,edit", [(False, False), (True, False), (False, True)],
                         ids=["fixed-schedule", "finishes-at-first-pass", "editing-guidance"])
def test_block_graph_matches_host_driven_block(early, edit):
    """dllm_block_graph_create captures a block (T_s passes, each inside a conditional node that runs it only while
    masked positions are left, then the commit pass). Launched from the same start it leaves the same tokens, mask,
    caches and step outputs as the passes called one by one from the host, launched twice in a row. With editing
    guidance the three row groups end with the same tokens."""
    w = scaled(SMALL, name="small-bf16-graph", mode=1, tau=0.0, k_max=32, T_s=6) if early else SMALL
    if edit:
        w = scaled(SMALL, name="small-bf16-graph-edit", B=3, cfg=2, cfg_scale=4.0, cfg_image_scale=1.5,
                   vocab_offset=1024 - 256, vocab_len=256)
    wt, caches, eng, _, _ = _setup(w, seed=43)
    tokens0, mask0 = eng.tokens.clone(), eng.mask.clone()
    caches0 = [(k.clone(), v.clone()) for k, v in caches]
    eng.decode_block()                         # host-driven reference (also warms the library's set-up)
    torch.cuda.synchronize()
    want = _snapshot(eng, caches)
    want_sel = (eng.sel.clone(), eng.nsel.clone(), eng.remaining.clone())
    g = eng.block_graph()
    assert g.conditional, g.note
    for _ in range(2):
        for (k, v), (k0, v0) in zip(caches, caches0):
            k.copy_(k0)
            v.copy_(v0)
        eng.set_block(tokens0, mask0)
        g.launch()
        torch.cuda.synchronize()
        assert bd.status_check(eng.ws) == bd.OK
        assert torch.equal(eng.tokens, want[0]) and torch.equal(eng.mask, want[1])
        for (k, v), (k1, v1) in zip(caches, want[2]):
            assert torch.equal(k, k1) and torch.equal(v, v1)
        if not early:     # with an early finish the graph skips passes whose step outputs the host loop rewrote
            assert torch.equal(eng.sel, want_sel[0]) and torch.equal(eng.nsel, want_sel[1])
        assert int(eng.remaining.item()) == 0 and int(eng.mask.sum().item()) == 0
        if edit:
            assert torch.equal(eng.tokens[0], eng.tokens[1]) and torch.equal(eng.tokens[0], eng.tokens[2])
    del g
