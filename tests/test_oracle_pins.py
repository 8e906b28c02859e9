"""Pins of the fp64 oracle against facts that do not come from the oracle itself: closed forms, library routines
on the special cases the method reduces to, brute force on tiny inputs, invariants, and the pages' schedule."""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import dllm_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


# ---------------------------------------------------------------------------------------------- storage rounding

def test_round_bf16_matches_torch_conversion():
    x = torch.randn(200000, dtype=torch.float32) * 3.0
    got = O.round_bf16(x.double().numpy())
    want = x.to(torch.bfloat16).double().numpy()
    assert np.array_equal(got, want)


def test_round_bf16_ties_to_even():
    # values exactly halfway between two bf16 neighbours: 1 + 2^-8 lies between 1 and 1 + 2^-7
    assert O.round_bf16(1.0 + 2.0 ** -8) == 1.0                      # even neighbour is 1.0
    assert O.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2 * 2.0 ** -7   # halfway, rounds up to even mantissa
    assert O.round_bf16(-(1.0 + 2.0 ** -8)) == -1.0
    assert O.round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7


# ---------------------------------------------------------------------------------------------- RMSNorm / SwiGLU

def test_rmsnorm_closed_forms():
    H, eps = 64, 1e-6
    for c in (0.5, -2.0, 3.25):
        y = O.rmsnorm(np.full((1, H), c), np.full(H, 2.0), eps)
        assert np.allclose(y, 2.0 * c / math.sqrt(c * c + eps), rtol=1e-15, atol=0)
    x = rng.standard_normal((3, H))
    g = rng.uniform(0.5, 1.5, H)
    y = O.rmsnorm(x, g, 0.0)
    assert np.allclose(np.sqrt(np.mean((y / g) ** 2, axis=1)), 1.0, atol=1e-14)
    assert np.allclose(O.rmsnorm(7.0 * x, g, 0.0), y, atol=1e-14)


def test_swiglu_closed_form():
    from scipy.special import expit
    H, I = 16, 8
    x = rng.standard_normal((2, H))
    wgu = rng.standard_normal((2 * I, H)) * 0.3
    wd = rng.standard_normal((H, I)) * 0.3
    gate, up = x @ wgu[:I].T, x @ wgu[I:].T
    want = (gate * expit(gate) * up) @ wd.T
    # storage in f32 perturbs by < 1e-7 relative
    got = O.swiglu_mlp(x, wgu, wd, "f32")
    assert np.allclose(got, want, rtol=1e-6, atol=1e-7)


# ---------------------------------------------------------------------------------------------- RoPE

def test_rope_d4_closed_form():
    # rotate-half pairing: element i pairs with i + d/2; angle = pos * base^(-2i/d)
    base = 100.0
    x = np.array([[[1.0, 2.0, 3.0, 4.0]]])     # [n=1, heads=1, d=4]
    p = 3.0
    a0, a1 = p * 1.0, p * base ** (-0.5)
    want = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
            3 * math.cos(a0) + 1 * math.sin(a0), 4 * math.cos(a1) + 2 * math.sin(a1)]
    assert np.allclose(O.rope(x, [p], base)[0, 0], want, atol=1e-14)
    assert np.allclose(O.rope(x, [0], base), x)


def test_rope_relative_position_and_norm():
    d = 32
    q = rng.standard_normal((5, 1, d))
    k = rng.standard_normal((5, 1, d))
    pq, pk = np.array([3, 7, 11, 50, 64]), np.array([0, 2, 9, 40, 64])
    s0 = np.einsum("nhd,mhd->nm", O.rope(q, pq, 1e4), O.rope(k, pk, 1e4))
    s1 = np.einsum("nhd,mhd->nm", O.rope(q, pq + 1000, 1e4), O.rope(k, pk + 1000, 1e4))
    assert np.allclose(s0, s1, atol=1e-10)
    assert np.allclose(np.linalg.norm(O.rope(k, pk, 1e4), axis=-1), np.linalg.norm(k, axis=-1), atol=1e-12)


# ---------------------------------------------------------------------------------------------- attention

def _sdpa(q, k, v, causal):
    """Library attention in fp64: q [L, Hq, d], k/v [N, Hkv, d] (GQA expanded by repeat_interleave)."""
    rep = q.shape[1] // k.shape[1]
    tq = torch.from_numpy(q).permute(1, 0, 2)
    tk = torch.from_numpy(k).repeat_interleave(rep, dim=1).permute(1, 0, 2)
    tv = torch.from_numpy(v).repeat_interleave(rep, dim=1).permute(1, 0, 2)
    return F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal).permute(1, 0, 2).numpy()


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2)])
def test_attention_one_block_is_full_bidirectional(Hq, Hkv):
    n, d = 12, 16
    q, k, v = (rng.standard_normal((n, h, d)) for h in (Hq, Hkv, Hkv))
    pos = np.arange(n)
    got = O.attention(q, k, v, pos, pos, blk_len=n)
    assert np.allclose(got, _sdpa(q, k, v, causal=False), atol=1e-12)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2)])
def test_attention_block_one_is_causal(Hq, Hkv):
    n, d = 10, 8
    q, k, v = (rng.standard_normal((n, h, d)) for h in (Hq, Hkv, Hkv))
    pos = np.arange(n)
    got = O.attention(q, k, v, pos, pos, blk_len=1)
    assert np.allclose(got, _sdpa(q, k, v, causal=True), atol=1e-12)


def test_attention_brute_force_tiny_block_causal():
    L, Lq, P, Hq, Hkv, d = 2, 4, 2, 2, 1, 3
    q = rng.standard_normal((Lq, Hq, d))
    k = rng.standard_normal((P + Lq, Hkv, d))
    v = rng.standard_normal((P + Lq, Hkv, d))
    qpos = np.arange(P, P + Lq)
    kpos = np.arange(P + Lq)
    got = O.attention(q, k, v, qpos, kpos, blk_len=L)
    for i in range(Lq):
        for h in range(Hq):
            ws, acc = [], np.zeros(d)
            for j in range(P + Lq):
                if kpos[j] // L <= qpos[i] // L:
                    ws.append((j, math.exp(sum(q[i, h, c] * k[j, 0, c] for c in range(d)) / math.sqrt(d))))
            tot = sum(wt for _, wt in ws)
            for j, wt in ws:
                acc += wt / tot * v[j, 0]
            assert np.allclose(got[i, h], acc, atol=1e-12)


def test_attention_decode_block_sees_whole_prefix():
    # queries are the last block: no key is hidden, so the result is unmasked attention over [prefix; block]
    P, L, Hq, Hkv, d = 64, 8, 4, 2, 16
    q = rng.standard_normal((L, Hq, d))
    k, v = rng.standard_normal((P + L, Hkv, d)), rng.standard_normal((P + L, Hkv, d))
    got = O.attention(q, k, v, np.arange(P, P + L), np.arange(P + L), blk_len=L)
    assert np.allclose(got, _sdpa(q, k, v, causal=False), atol=1e-12)


def test_attention_thinned_equals_full_with_dropped_keys_removed_from_softmax():
    P, L, H, d = 40, 8, 2, 8
    q = rng.standard_normal((L, H, d))
    k, v = rng.standard_normal((P + L, H, d)), rng.standard_normal((P + L, H, d))
    keep = np.sort(rng.choice(P, 17, replace=False))
    kpos = np.concatenate([keep, np.arange(P, P + L)])
    got = O.attention(q, k[kpos], v[kpos], np.arange(P, P + L), kpos, blk_len=L)
    # full key set, with an additive mask of -inf on the dropped keys, through the library routine
    tq = torch.from_numpy(q).permute(1, 0, 2)
    tk = torch.from_numpy(k).permute(1, 0, 2)
    tv = torch.from_numpy(v).permute(1, 0, 2)
    m = torch.full((L, P + L), float("-inf"), dtype=torch.float64)
    m[:, torch.from_numpy(kpos)] = 0.0
    want = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=m).permute(1, 0, 2).numpy()
    assert np.allclose(got, want, atol=1e-12)


def test_attention_rope_shift_invariance_on_thinned_set():
    P, L, H, d = 32, 8, 2, 16
    qr = rng.standard_normal((L, H, d))
    kr, v = rng.standard_normal((P + L, H, d)), rng.standard_normal((P + L, H, d))
    keep = np.sort(rng.choice(P, 11, replace=False))
    kpos = np.concatenate([keep, np.arange(P, P + L)])
    qpos = np.arange(P, P + L)
    a = O.attention(O.rope(qr, qpos, 1e4), O.rope(kr[kpos], kpos, 1e4), v[kpos], qpos, kpos, L)
    # shift by a multiple of L so the block structure is unchanged
    s = 5 * L
    b = O.attention(O.rope(qr, qpos + s, 1e4), O.rope(kr[kpos], kpos + s, 1e4), v[kpos], qpos + s, kpos + s, L)
    assert np.allclose(a, b, atol=1e-10)


# ---------------------------------------------------------------------------------------------- SPRINT retention

def test_prefix_scores_invariant_under_rope():
    Hkv, P, d = 4, 48, 16
    k = rng.standard_normal((Hkv, P, d))
    kr = O.rope(k.transpose(1, 0, 2), np.arange(P), 1e4).transpose(1, 0, 2)
    assert np.allclose(O.prefix_scores(k), O.prefix_scores(kr), atol=1e-12)
    assert abs(O.prefix_scores(k).mean() - 1.0) < 1e-14


def test_prefix_scores_hand_computed_mean_of_head_norms():
    """Hand-computed case in which the mean over kv heads of the per-head l2 norms ranks the positions differently
    from the squared norm, the l2 norm of the whole key (all heads), the largest head norm and the l1 norm.
    Head vectors (kv head 0 | kv head 1):
      position 0: (3, 4) | (0, 0)    head norms 5, 0     -> mean 2.5   (l1 mean 3.5, max 5, squared mean 12.5)
      position 1: (2, 0) | (0, 3.5)  head norms 2, 3.5   -> mean 2.75  (l1 mean 2.75, max 3.5, squared mean 8.125)
      position 2: (0, 0) | (1, 0)    head norms 0, 1     -> mean 0.5
    Mean over the prefix = 5.75 / 3, so the normalised scores are 30/23, 33/23, 6/23, and keeping one position
    keeps position 1 (every alternative form listed would keep position 0)."""
    k = np.zeros((2, 3, 2))
    k[0, 0] = (3, 4)
    k[0, 1] = (2, 0)
    k[1, 1] = (0, 3.5)
    k[1, 2] = (1, 0)
    sc = O.prefix_scores(k)
    assert np.allclose(sc, [30 / 23, 33 / 23, 6 / 23], rtol=0, atol=1e-15)
    keep1, _, margin = O.prefix_retain(k, None, n_keep=1)
    assert list(keep1) == [1] and abs(margin - 3 / 23) < 1e-15
    keep2, _, _ = O.prefix_retain(k, 2 / 3)
    assert list(keep2) == [0, 1]


def test_prefix_retain_brute_force_and_ties():
    Hkv, P, d = 2, 9, 4
    k = rng.standard_normal((Hkv, P, d))
    k[:, 5] = k[:, 2]                    # planted exact tie between positions 2 and 5
    k[:, 7] = k[:, 2]
    sc = O.prefix_scores(k)
    for ratio in (0.1, 0.3, 0.5, 0.7, 1.0):
        keep, _, _ = O.prefix_retain(k, ratio)
        n = math.ceil(ratio * P)
        assert len(keep) == n and list(keep) == sorted(keep)
        # brute force over all subsets of size n: the kept set is the best by (score desc, position asc)
        import itertools
        best = min(itertools.combinations(range(P), n),
                   key=lambda s: sorted([(-sc[i], i) for i in s]))
        assert tuple(keep) == tuple(sorted(best))


# ---------------------------------------------------------------------------------------------- router / MoE

def _experts(H=12, I=6, E=5):
    wgu = rng.standard_normal((E, 2 * I, H)) * 0.3
    wd = rng.standard_normal((E, H, I)) * 0.3
    return wgu, wd


def test_router_all_experts_zero_bias_is_dense_soft_mixing():
    from scipy.special import expit
    T, H, E = 3, 12, 5
    h = rng.standard_normal((T, H))
    wr = rng.standard_normal((E, H)) * 0.5
    wgu, wd = _experts(E=E)
    ids, gates, s, _ = O.route(h, wr, np.zeros(E), E)
    got = O.moe_delta(h, ids, gates, wgu, wd, None, None, "f32")
    # dense mixing written directly: sum_e sigmoid(l_e)/sum(sigmoid) * MLP_e(h)
    logits = h @ wr.T
    w = expit(logits)
    w = w / w.sum(axis=1, keepdims=True)
    I = wgu.shape[1] // 2
    mlp = np.stack([((h @ wgu[e, :I].T) * expit(h @ wgu[e, :I].T) * (h @ wgu[e, I:].T)) @ wd[e].T
                    for e in range(E)], axis=1)                      # [T, E, H]
    want = np.einsum("te,teh->th", w, mlp)
    assert np.allclose(got, want, rtol=1e-6, atol=1e-7)


def test_single_expert_top1_is_one_mlp_plus_shared():
    T, H = 4, 12
    h = rng.standard_normal((T, H))
    wgu, wd = _experts(E=1)
    sgu, sd = _experts(E=1)
    ids, gates, _, _ = O.route(h, rng.standard_normal((1, H)), np.zeros(1), 1)
    assert np.all(ids == 0) and np.allclose(gates, 1.0)
    got = O.moe_delta(h, ids, gates, wgu, wd, sgu[0], sd[0], "f32")
    want = O.swiglu_mlp(h, wgu[0], wd[0], "f32") + O.swiglu_mlp(h, sgu[0], sd[0], "f32")
    assert np.allclose(got, want, atol=1e-12)


def test_bias_forces_selection_but_not_gates():
    T, H, E, k = 6, 16, 10, 3
    h = rng.standard_normal((T, H))
    wr = rng.standard_normal((E, H))
    bias = np.zeros(E)
    forced = [7, 2, 4]
    bias[forced] = [30.0, 20.0, 10.0]
    ids, gates, s, _ = O.route(h, wr, bias, k)
    for t in range(T):
        assert list(ids[t]) == forced                       # slots in biased-score order
        sel = s[t, forced]
        assert np.allclose(gates[t], sel / sel.sum())        # gates from the unbiased sigmoid scores
        assert abs(gates[t].sum() - 1.0) < 1e-14


def test_router_ties_lower_expert_wins():
    h = np.zeros((1, 4))                                     # every sigmoid score is 0.5
    ids, gates, _, margin = O.route(h, np.ones((6, 4)), np.zeros(6), 2)
    assert list(ids[0]) == [0, 1] and np.allclose(gates, 0.5) and margin[0] == 0.0


def test_router_margins_set_and_order():
    """Hand-built biased scores: the set margin is the gap between slot k-1 and the best unchosen expert; the
    order margin is the smallest gap between consecutive biased scores among the best k + 1."""
    # zero router weights: every score is sigmoid(0) = 1/2, so the biased scores are 1/2 + bias
    bias = np.array([0.30, 0.10, 0.29, -0.2, 0.05])
    h = np.zeros((1, 3))
    ids, gates, s, set_m = O.route(h, np.zeros((5, 3)), bias, 2)
    _, _, _, ord_m = O.route(h, np.zeros((5, 3)), bias, 2, order=True)
    assert list(ids[0]) == [0, 2] and np.allclose(gates, 0.5)
    assert abs(set_m[0] - 0.19) < 1e-12          # 0.79 - 0.60
    assert abs(ord_m[0] - 0.01) < 1e-12          # 0.80 - 0.79 (slots 0 and 1 nearly swap)


def test_moe_permutation_equivariance():
    T, H, E, k = 5, 12, 5, 2
    h = rng.standard_normal((T, H))
    wr = rng.standard_normal((E, H))
    b = rng.uniform(-0.1, 0.1, E)
    wgu, wd = _experts(E=E)
    ids, g, _, _ = O.route(h, wr, b, k)
    out = O.moe_delta(h, ids, g, wgu, wd, None, None, "f32")
    p = rng.permutation(T)
    ids2, g2, _, _ = O.route(h[p], wr, b, k)
    out2 = O.moe_delta(h[p], ids2, g2, wgu, wd, None, None, "f32")
    assert np.allclose(out[p], out2, atol=1e-14)


# ---------------------------------------------------------------------------------------------- confidence / unmask

def test_confidence_equal_logits_is_one_over_v():
    for V in (7, 1024, 157184):
        cand, c, _, _ = O.confidence(np.full((1, V), 0.375))
        assert cand[0] == 0 and abs(c[0] - 1.0 / V) < 1e-15 / V * 10


def test_confidence_single_spike_closed_form():
    V = 4096
    for delta, at in ((3.0, 17), (0.5, 4095), (12.0, 0)):
        z = np.zeros((1, V))
        z[0, at] = delta
        cand, c, _, _ = O.confidence(z)
        assert cand[0] == at
        assert abs(c[0] - math.exp(delta) / (math.exp(delta) + V - 1)) < 1e-15


def test_confidence_brute_force_small_vocab():
    for V in (2, 5, 16):
        z = np.round(rng.standard_normal((4, V)) * 2, 1)
        z[0, 3 % V] = z[0, 1 % V] = z[0].max() + 1          # planted tie for the argmax
        cand, c, lse, _ = O.confidence(z)
        for r in range(4):
            ex = [math.exp(float(v)) for v in z[r]]
            best = max(range(V), key=lambda i: (z[r, i], -i))
            assert cand[r] == best
            assert abs(c[r] - max(ex) / sum(ex)) < 1e-14
            assert abs(lse[r] - math.log(sum(ex))) < 1e-12


def test_fixed_schedule_golden():
    g = json.load(open(os.path.join(GOLDEN, "schedule.json")))
    for case in g["cases"]:
        m, ks = case["L"], []
        for t in range(case["T_s"]):
            k = O.unmask_count(m, t, case["T_s"], 0)
            ks.append(k)
            m -= k
        assert ks == case["k_per_step"], case["cite"]
        assert m == 0


def _run_block(L, T_s, mode, tau, k_max, conf_fn):
    m, ks = L, []
    for t in range(T_s):
        c = conf_fn(t, m)
        k = O.unmask_count(m, t, T_s, mode, tau, k_max, c)
        ks.append(k)
        m -= k
    return ks, m


@pytest.mark.parametrize("mode", [0, 1])
def test_block_finishes_on_the_last_step(mode):
    for trial in range(50):
        L, T_s = int(rng.integers(1, 65)), int(rng.integers(1, 40))
        ks, m = _run_block(L, T_s, mode, 0.9, 8, lambda t, m: rng.uniform(0.5, 1.0, m))
        assert m == 0 and sum(ks) == L
        # the last step that unmasks anything is the last step when the schedule is tight
        if mode == 0 and T_s <= L:
            assert all(k > 0 for k in ks)


def test_threshold_limits():
    L, T_s = 32, 32
    ks, _ = _run_block(L, T_s, 1, 1.0, 8, lambda t, m: rng.uniform(0.0, 1.0, m))   # tau >= 1: nothing exceeds
    assert ks == [O.unmask_count(L - sum(ks[:t]), t, T_s, 0) for t in range(T_s)]
    ks, _ = _run_block(L, T_s, 1, -1.0, 8, lambda t, m: rng.uniform(0.0, 1.0, m))  # tau below every c
    assert ks[:4] == [8, 8, 8, 8] and sum(ks) == L


def test_unmask_selection_and_writeback():
    B, L, V = 2, 6, 11
    tokens = np.full((B, L), 99)
    mask = np.ones((B, L), dtype=np.int64)
    mask[1, 2] = 0
    tokens[1, 2] = 5
    row_pos = np.nonzero(mask.reshape(-1))[0]
    z = rng.standard_normal((len(row_pos), V))
    u = O.unmask(z, row_pos, tokens, mask, t=0, T_s=3, mode=0)
    for b in range(B):
        m = int(mask[b].sum())
        k = -(-m // 3)
        assert u["nsel"][b] == k and len(u["sel"][b]) == k
        c = u["conf"][b]
        chosen = set(u["sel"][b])
        rest = [i for i in range(L) if mask[b, i] and i not in chosen]
        assert all(c[i] >= c[j] for i in chosen for j in rest)
        for i in chosen:
            assert u["mask"][b, i] == 0 and u["tokens"][b, i] == u["cand"][b, i]
    assert u["tokens"][1, 2] == 5 and u["mask"][1, 2] == 0


def test_cfg3_reduces_to_two_way_guidance():
    """Editing guidance against the two-way formula and the rows themselves (float32-representable inputs, so every
    case below is exact in fp64): an image-only row equal to the unconditional one leaves text guidance of the full
    row; text scale 0 leaves image guidance between the image-only and the unconditional rows; an image-only row
    equal to the full row leaves two-way guidance with the image scale; both scales 1 give the full row."""
    zc = rng.standard_normal((3, 40)).astype(np.float32).astype(np.float64)
    zi = rng.standard_normal((3, 40)).astype(np.float32).astype(np.float64)
    zu = rng.standard_normal((3, 40)).astype(np.float32).astype(np.float64)
    assert np.array_equal(O.cfg3_combine(zc, zu, zu, 2.5, 1.5), O.cfg_combine(zc, zu, 2.5))
    assert np.array_equal(O.cfg3_combine(zc, zi, zu, 0.0, 1.5), O.cfg_combine(zi, zu, 1.5))
    assert np.array_equal(O.cfg3_combine(zc, zc, zu, 2.5, 1.5), O.cfg_combine(zc, zu, 1.5))
    assert np.array_equal(O.cfg3_combine(zc, zi, zu, 1.0, 1.0), zc)


def test_cfg3_fp32_error_bound_covers_float32_evaluation():
    """The bound covers a float32 evaluation in the stated order, each operation rounded to nearest, on rows with
    large and cancelling logits."""
    g = np.random.default_rng(7)
    zc = (g.standard_normal((64, 300)) * 20).astype(np.float32)
    zi = (zc + g.standard_normal((64, 300)).astype(np.float32) * 0.5).astype(np.float32)
    zu = (g.standard_normal((64, 300)) * 20).astype(np.float32)
    for st, si in ((4.0, 1.5), (1.0, 1.0), (7.5, 0.25)):
        st32, si32 = np.float32(st), np.float32(si)
        a = zu + si32 * (zi - zu)
        z32 = (a + st32 * (zc - zi)).astype(np.float64)
        err = np.abs(z32 - O.cfg3_combine(zc, zi, zu, st, si)).max(axis=1)
        assert np.all(err <= O.cfg3_fp32_error_bound(zc, zi, zu, st, si))


def test_unmask_editing_guidance_updates_every_third():
    """With three rows per position the chosen token is written to the position in all three thirds of the batch,
    and the choice is that of the guided logits."""
    B, L, V = 6, 4, 10   # 2 logical rows
    mask = np.ones((B, L), dtype=np.int64)
    tokens = np.full((B, L), V - 1, dtype=np.int64)
    row_pos = np.arange(2 * L)
    g = np.random.default_rng(3)
    zc, zi, zu = (g.standard_normal((2 * L, V)) for _ in range(3))
    u = O.unmask(zc, row_pos, tokens, mask, t=0, T_s=2, mode=0, k_max=8, z_uncond=zu, cfg_scale=3.0, z_image=zi,
                 cfg_image_scale=1.5)
    z = O.cfg3_combine(zc, zi, zu, 3.0, 1.5)
    for b in range(2):
        for i in u["sel"][b]:
            want = int(np.argmax(z[b * L + i]))
            for grp in range(3):
                assert u["tokens"][b + 2 * grp, i] == want and u["mask"][b + 2 * grp, i] == 0


def test_cfg_combine_special_scales():
    zc = rng.standard_normal((3, 50)).astype(np.float32).astype(np.float64)
    zu = rng.standard_normal((3, 50)).astype(np.float32).astype(np.float64)
    # scale 0 is the unconditional row, scale 1 the conditional one, scale 2 the extrapolation 2 z_c - z_u
    # (all exact in fp64 for float32 inputs)
    assert np.array_equal(O.cfg_combine(zc, zu, 0.0), zu)
    assert np.array_equal(O.cfg_combine(zc, zu, 1.0), zc)
    assert np.array_equal(O.cfg_combine(zc, zu, 2.0), 2 * zc - zu)
    assert np.array_equal(O.cfg_combine(zc, zu, 0.5), 0.5 * (zc + zu))


def test_cfg_fp32_error_bound_covers_float32_evaluation():
    """The bound holds for a float32 evaluation (subtract, multiply, add, each rounded to nearest) at several
    scales and magnitudes, and is tight to within a small factor (it is not vacuous)."""
    worst = 0.0
    for scale in (2.0, 1.5, 3.7, 0.3):
        for mag in (1.0, 8.0, 100.0):
            zc = (rng.standard_normal((4, 4096)) * mag).astype(np.float32)
            zu = (rng.standard_normal((4, 4096)) * mag).astype(np.float32)
            s32 = np.float32(scale)
            fl = (zu + s32 * (zc - zu).astype(np.float32)).astype(np.float32).astype(np.float64)
            exact = O.cfg_combine(zc, zu, float(s32))
            err = np.abs(fl - exact).max(axis=1)
            bound = O.cfg_fp32_error_bound(zc, zu, float(s32))
            assert np.all(err <= bound)
            worst = max(worst, float((err / bound).max()))
    assert worst > 0.05


def test_unmask_flags_guided_candidate_ties():
    """Two candidates whose guided logits differ by less than the float32 rounding bound are flagged; a clear gap
    is not; without guidance nothing is flagged as a candidate tie."""
    V = 64
    zc = np.zeros((2, V))
    zu = np.zeros((2, V))
    zc[0, 3], zc[0, 9] = 10.0, 10.0 + 2.0 ** -20     # guided gap 2^-19, inside the bound at |z| ~ 20
    zc[1, 3], zc[1, 9] = 10.0, 10.5
    tok = np.full((2, 4), V - 1)
    msk = np.ones((2, 4), dtype=np.int64)
    u = O.unmask(zc, [0, 1], tok, msk, 0, 4, z_uncond=zu, cfg_scale=2.0)
    assert u["tie_cand"][0, 0] and not u["tie_cand"][0, 1]
    assert u["cand"][0, 0] == 9 and u["cand"][0, 1] == 9
    u0 = O.unmask(zc, [0, 1], tok[:1], msk[:1], 0, 4)
    assert not u0["tie_cand"].any() and np.all(u0["conf_rtol"] == 1e-6)


# ---------------------------------------------------------------------------------------------- composition

def test_forward_block_matches_textbook_layer_in_torch():
    """One layer over P=0 with the block covering the whole sequence is a textbook pre-norm transformer layer
    with a sigmoid-routed MoE FFN; written here with torch library ops in fp64 (no storage rounding)."""
    from block_diffusion_moe_dllm_b200.configs import TINY_F32, scaled
    from block_diffusion_moe_dllm_b200 import synth
    w = scaled(TINY_F32, H=32, Hq=4, Hkv=2, d=8, E=4, k=2, I=16, V=64, P=16, L=8, seed=3)
    wt = synth.make_weights(w, random_gains=True)
    caches = synth.make_prefix_cache(w)
    tokens, mask = synth.make_block_state(w, masked_fraction=0.6)
    f = O.forward_block(w, wt, caches, tokens.numpy(), mask.numpy())

    d64 = lambda a: a.double()
    lw = wt["layers"][0]
    tok = torch.where(mask.bool(), torch.full_like(tokens, w.mask_id), tokens).reshape(-1).long()
    x = d64(wt["embed"])[tok]
    h = F.rms_norm(x, (w.H,), d64(lw["attn_norm"]), w.eps)
    qkv = h @ d64(lw["w_qkv"]).T
    q = qkv[:, : w.Hq * w.d].reshape(w.L, w.Hq, w.d)
    k = qkv[:, w.Hq * w.d: (w.Hq + w.Hkv) * w.d].reshape(w.L, w.Hkv, w.d)
    v = qkv[:, (w.Hq + w.Hkv) * w.d:].reshape(w.L, w.Hkv, w.d)
    pos = torch.arange(w.P, w.P + w.L, dtype=torch.float64)
    inv = w.rope_base ** (-torch.arange(0, w.d, 2, dtype=torch.float64) / w.d)
    ang = pos[:, None] * inv[None, :]
    cos = torch.cat([ang.cos(), ang.cos()], -1)[:, None]
    sin = torch.cat([ang.sin(), ang.sin()], -1)[:, None]
    rot = lambda t: torch.cat([-t[..., w.d // 2:], t[..., : w.d // 2]], -1)
    q, k = q * cos + rot(q) * sin, k * cos + rot(k) * sin
    kc, vc = d64(caches[0][0][0, :, : w.P]).permute(1, 0, 2), d64(caches[0][1][0, :, : w.P]).permute(1, 0, 2)
    K, Vv = torch.cat([kc, k]), torch.cat([vc, v])
    o = F.scaled_dot_product_attention(q.permute(1, 0, 2), K.permute(1, 0, 2), Vv.permute(1, 0, 2),
                                       enable_gqa=True).permute(1, 0, 2).reshape(w.L, -1)
    x = x + o @ d64(lw["w_o"]).T
    h2 = F.rms_norm(x, (w.H,), d64(lw["ffn_norm"]), w.eps)
    s = torch.sigmoid(h2 @ d64(lw["w_router"]).T)
    top = torch.topk(s + d64(lw["router_bias"]), w.k, dim=1).indices
    g = torch.gather(s, 1, top)
    g = g / g.sum(1, keepdim=True)

    def mlp(xx, gu, dn):
        a, b = (xx @ gu.T).chunk(2, dim=-1)
        return (F.silu(a) * b) @ dn.T
    y = mlp(h2, d64(lw["w_gu_shared"]), d64(lw["w_down_shared"]))
    for t in range(w.L):
        for j in range(w.k):
            e = int(top[t, j])
            y[t] += g[t, j] * mlp(h2[t], d64(lw["w_gu"][e]), d64(lw["w_down"][e]))
    x = x + y
    xf = F.rms_norm(x, (w.H,), d64(wt["final_norm"]), w.eps)
    rows = torch.nonzero(mask.reshape(-1)).reshape(-1)
    logits = xf[rows] @ d64(wt["w_lm"]).T
    assert np.allclose(f["x"].reshape(w.L, w.H), x.numpy(), rtol=1e-5, atol=1e-5)
    assert np.allclose(f["logits"], logits.numpy(), rtol=1e-5, atol=1e-5)
    assert np.array_equal(np.sort(f["route"][0][0], axis=1), np.sort(top.numpy(), axis=1))


def test_denoise_block_end_to_end_tiny():
    """A full block: T_s passes then the commit pass; every position ends unmasked and k_t follows the schedule."""
    from block_diffusion_moe_dllm_b200.configs import TINY_F32, scaled
    from block_diffusion_moe_dllm_b200 import synth
    w = scaled(TINY_F32, H=32, Hq=4, Hkv=2, d=8, E=4, k=2, I=16, V=64, P=16, L=8, T_s=3, seed=5)
    wt = synth.make_weights(w)
    caches = synth.make_prefix_cache(w)
    tokens, mask = synth.make_block_state(w)
    tokens, mask = tokens.numpy(), mask.numpy()
    for t in range(w.T_s):
        u = O.denoise_step(w, wt, caches, tokens, mask, t)
        tokens, mask = u["tokens"], u["mask"]
    assert mask.sum() == 0 and np.all(tokens < w.V)
    bk, bv = O.commit_block(w, wt, caches, tokens)
    assert len(bk) == w.n_layers and bk[0].shape == (w.B, w.L, w.Hkv, w.d)


# ---------------------------------------------------------------------------------------------- FP8 weights

def test_e4m3_values_match_torch_conversion_for_every_code():
    """All 256 E4M3 codes decode to torch's float8_e4m3fn values (the same OCP format), NaN codes included."""
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_value(codes)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])


def test_e4m3_closed_forms():
    v = O.e4m3_value(np.array([0x00, 0x80, 0x38, 0xB8, 0x7E, 0x01, 0x08, 0x3C, 0x7F]))
    assert v[0] == 0.0 and v[1] == 0.0 and np.signbit(v[1])
    assert v[2] == 1.0 and v[3] == -1.0            # exponent 7 = bias, mantissa 0
    assert v[4] == 448.0                           # largest finite: 2^8 * 1.75
    assert v[5] == 2.0 ** -9                       # smallest subnormal: 2^-6 * 1/8
    assert v[6] == 2.0 ** -6                       # smallest normal
    assert v[7] == 1.5
    assert np.isnan(v[8])


def test_dequant_rows_scales_each_output_row():
    q = np.array([[0x38, 0xB8], [0x40, 0x30]], dtype=np.uint8)      # [[1, -1], [2, 0.5]]
    w = O.dequant_rows(q, np.array([0.5, 3.0], dtype=np.float32))
    assert np.array_equal(w, [[0.5, -0.5], [6.0, 1.5]])


# ---------------------------------------------------------------------------------------------- position scores

def test_position_scores_closed_forms():
    V = 50
    zu = np.zeros((1, V))                            # uniform: p = 1/V everywhere
    assert abs(O.position_scores(zu, "low_confidence")[0] - 1 / V) < 1e-15
    assert abs(O.position_scores(zu, "top_k_margin")[0]) < 1e-15
    assert abs(O.position_scores(zu, "neg_entropy")[0] + math.log(V)) < 1e-12
    d = 3.0                                          # one spike: p1 = e^d / (e^d + V - 1), the rest 1 / (e^d + V - 1)
    zs = np.zeros((1, V))
    zs[0, 7] = d
    S = math.exp(d) + V - 1
    p1, p0 = math.exp(d) / S, 1 / S
    assert abs(O.position_scores(zs, "top_k_margin")[0] - (p1 - p0)) < 1e-15
    ent = p1 * math.log(p1) + (V - 1) * p0 * math.log(p0)
    assert abs(O.position_scores(zs, "neg_entropy")[0] - ent) < 1e-12
    z2 = np.zeros((1, V))                            # the largest logit twice: margin 0
    z2[0, 3] = z2[0, 9] = 2.0
    assert O.position_scores(z2, "top_k_margin")[0] == 0.0


def test_position_scores_brute_force_small_vocab():
    for _ in range(20):
        z = rng.standard_normal((3, 7)) * 2
        p = np.exp(z) / np.exp(z).sum(axis=1, keepdims=True)
        srt = np.sort(p, axis=1)
        assert np.allclose(O.position_scores(z, "top_k_margin"), srt[:, -1] - srt[:, -2], atol=1e-15)
        assert np.allclose(O.position_scores(z, "neg_entropy"), (p * np.log(p)).sum(axis=1), atol=1e-13)
        assert np.allclose(O.position_scores(z, "low_confidence"), p.max(axis=1), atol=1e-15)


def test_unmask_ranks_by_score_and_counts_by_probability():
    """The strategies rank differently: position 0 (p = 0.60, 0.39, ...) has the larger top probability, position 1
    (p = 0.55, 0.05, ...) the larger margin and the lower entropy. The threshold count always uses the largest
    probability (here none exceeds tau, so one position per step is taken)."""
    V = 10
    pa = np.array([0.60, 0.39] + [0.01 / 8] * 8)
    pb = np.array([0.55] + [0.05] * 9)
    z = np.log(np.stack([pa, pb]))
    tok = np.full((1, 2), V - 1)
    msk = np.ones((1, 2), dtype=np.int64)
    args = dict(mode=1, tau=0.9, k_max=2)
    assert list(O.unmask(z, [0, 1], tok, msk, 0, 2, score="low_confidence", **args)["sel"][0]) == [0]
    assert list(O.unmask(z, [0, 1], tok, msk, 0, 2, score="top_k_margin", **args)["sel"][0]) == [1]
    ent_a, ent_b = (pa * np.log(pa)).sum(), (pb * np.log(pb)).sum()
    assert ent_b < ent_a                     # position 0 has the lower entropy: neg_entropy ranks it first
    assert list(O.unmask(z, [0, 1], tok, msk, 0, 2, score="neg_entropy", **args)["sel"][0]) == [0]
    u = O.unmask(z, [0, 1], tok, msk, 0, 2, score="top_k_margin", **args)
    assert np.allclose(u["rank"][0], [0.60 - 0.39, 0.55 - 0.05]) and np.allclose(u["conf"][0], [0.60, 0.55])


# ---------------------------------------------------------------------------------------------- SPRINT mixed score

def test_prefix_importance_mixes_key_norm_and_confidence():
    """s = alpha l~ + (1 - alpha) c: alpha = 1 is the key-norm term, alpha = 0 the confidence alone, alpha = 0.5
    their mean (the hand-computed key norms of the kv-head pin: 30/23, 33/23, 6/23)."""
    k = np.zeros((2, 3, 2))
    k[0, 0] = (3, 4)
    k[0, 1] = (2, 0)
    k[1, 1] = (0, 3.5)
    k[1, 2] = (1, 0)
    c = np.array([0.9, 0.1, 0.5])
    assert np.allclose(O.prefix_importance(k, c, 1.0), [30 / 23, 33 / 23, 6 / 23], atol=1e-15)
    assert np.allclose(O.prefix_importance(k, c, 0.0), c, atol=1e-15)
    half = O.prefix_importance(k, c, 0.5)
    assert np.allclose(half, [0.5 * 30 / 23 + 0.45, 0.5 * 33 / 23 + 0.05, 0.5 * 6 / 23 + 0.25], atol=1e-15)
    keep, _, _ = O.prefix_retain(k, None, n_keep=1, conf=c, alpha=0.5)
    assert list(keep) == [0]          # 1.102 > 0.767 > 0.380: the confidence moves the choice from 1 to 0


def test_prefix_retain_per_modality_counts_brute_force():
    """With a modality mask, n_keep_img image positions and n_keep - n_keep_img text positions are kept, each the
    best of its modality (brute force over subsets), in position order."""
    import itertools
    Hkv, P, d = 2, 10, 4
    k = rng.standard_normal((Hkv, P, d))
    c = rng.uniform(size=P)
    mod = np.array([1, 1, 0, 1, 0, 1, 1, 0, 0, 1])
    sc = O.prefix_importance(k, c, 0.5)
    for n_img, n_txt in [(3, 2), (6, 0), (0, 4), (2, 4)]:   # the mask has 6 image and 4 text positions
        keep, _, _ = O.prefix_retain(k, None, n_keep=n_img + n_txt, conf=c, alpha=0.5, modality=mod,
                                     n_keep_img=n_img)
        assert len(keep) == n_img + n_txt and list(keep) == sorted(keep)
        assert int(mod[keep].sum()) == n_img
        img = [i for i in range(P) if mod[i]]
        best = max(itertools.combinations(img, n_img), key=lambda s: sorted([sc[i] for i in s]))
        assert set(best) == {i for i in keep if mod[i]}


def test_prefix_retain_modality_shortfall_moves_to_the_other_modality():
    k = rng.standard_normal((1, 6, 4))
    mod = np.array([1, 0, 1, 0, 0, 0])                # 2 image, 4 text positions
    keep, _, _ = O.prefix_retain(k, None, n_keep=5, modality=mod, n_keep_img=4)
    assert len(keep) == 5 and set(keep) >= {0, 2}      # both images kept, 3 of the 4 text positions
    keep, _, _ = O.prefix_retain(k, None, n_keep=5, modality=mod, n_keep_img=0)
    assert len(keep) == 5 and len(set(keep) & {0, 2}) == 1   # 4 text positions, then one image
