"""Plain fp64 CPU oracle for one block-diffusion denoising step of the LLaDA2.0-Uni MoE dLLM backbone.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import this module. The library (CUDA kernels behind the C ABI and its Python binding) never
calls it and shares no code with it.

Every step is its plain definition, in fp64 numpy, in the pages' order. Sources, by page title and section:

  [R] "[논문 리뷰] LLaDA2.0-Uni: Unifying Multimodal Understanding and Generation with Diffusion Large Language
      Model" (paper review, baba9811.github.io):
        "Block Diffusion Language Model (BDLM)"  - blocks: bidirectional inside, left-to-right across, earlier
                                                   blocks always clean context
        "MoE 백본과 Block-wise Attention"          - MoE backbone, router picks top-k experts per token; block-wise
                                                   attention pattern
        "Positional Embedding & 임의 해상도"       - 1D RoPE over the flattened sequence
        "SPRINT — 학습 없는 추론 가속"              - sparse prefix retention (mean-normalised key norm l~_i,
                                                   alpha = 0.5, per-modality keep ratios); non-uniform unmasking
                                                   (accept all c > tau ~ 0.93, at least ceil(m/(T-t)) per step;
                                                   the standard schedule ceil(m/T)); c_i = max_v p(v | x_t)
        "BDLM Loss (사전학습)"                     - conditioning on clean x_{0,<k} and noisy x_{t,k}
        "Load Balancing — Auxiliary-loss-free MoE Bias" - a per-expert bias steers expert load
  [M] "LLaDA2.0-Uni：基于扩散大型语言模型的多模态理解与生成统一框架" (HF-mirror README, ai.gitcode.com):
        "SPRINT 加速技术"  - prefix KV computed once in a warm-up and reused; adaptive unmasking with
                           k = ceil(remaining_masked / steps_left); batch acceptance of all p > threshold;
                           keep_ratio / cache_warmup_steps knobs
        usage examples     - block_length=32, steps=8, cfg_scale=2.0 (text-to-image); steps=32,
                             threshold=0.93, keep_ratio=0.5 (understanding)

Readings where the pages are silent (each also listed in the design notes):
  * router: sigmoid scores; bias added for selection only; gates = unbiased scores of the chosen experts,
    renormalised to sum 1; no extra routed scaling; ties -> lower expert id; slots ordered by biased score.
  * shared expert: same SwiGLU MLP on every token, weight 1.
  * SwiGLU: down(silu(gate x) * (up x)); fused gate|up weight stores gate rows then up rows.
  * RMSNorm: x / sqrt(mean(x^2) + eps) * g.
  * RoPE: rotate-half pairing (i, i + d/2), theta_i = base^(-2i/d), absolute positions.
  * attention: scale 1/sqrt(d); kv head of q head h is floor(h * Hkv / Hq); key j visible to query i iff
    floor(pos_j / L) <= floor(pos_i / L).
  * SPRINT score (formula stripped on the page): key-norm term only, l_i = mean over kv heads of ||K[h, i]||_2,
    divided by its mean over the prefix; keep ceil(r * P) largest, ties -> lower position; kept set in
    position order.
  * threshold rule (formula stripped on the page): k_t = min(m, max(ceil(m / (T_s - t)), min(k_max, #{c > tau}))).
  * CFG: z = z_u + s (z_c - z_u), s = cfg_scale, in fp64; decisions within the float32 rounding bound of that
    formula are flagged as near-ties (cfg_fp32_error_bound).
  * editing CFG (three rows per position, formula not printed): z = z_u + s_i (z_i - z_u) + s_t (z_c - z_i), with
    s_t = cfg_text_scale (cfg_scale here) and s_i = cfg_image_scale; rows (b, b + B/3, b + 2B/3) are (instruction
    and image, image only, unconditional); near-ties by cfg3_fp32_error_bound.
  * confidence c = max softmax at temperature 1 over the scored vocabulary; candidate = lowest argmax.
  * storage rounding: wherever the library stores a tensor in its storage type (bf16 or fp32) the oracle rounds
    its fp64 value to that type (round-to-nearest-even) at the same point; between those points it is fp64.
"""
import math
import numpy as np

# --------------------------------------------------------------------------------------------------------------
# storage rounding


def round_bf16(x):
    """Round fp64 values to the nearest bf16 (8 significant bits, ties to even), returned as fp64."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def round_f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def store(x, dtype):
    """Value of ``x`` after the library writes it in storage type ``dtype`` ("bf16" or "f32")."""
    return round_bf16(x) if dtype == "bf16" else round_f32(x)


def f64(a):
    """Exact widening of a numpy array or torch tensor (bf16 / fp32 / int) to fp64 numpy."""
    if hasattr(a, "detach"):                 # torch tensor: widen through torch (exact), then to numpy
        import torch
        return a.detach().to("cpu", torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------------------------------------------
# FP8 weights (the FP8 checkpoint of the card news "FP8 추론" and the HF-mirror README's FP8 version: format not
# given on the pages; read as OCP FP8 E4M3 codes with one fp32 scale per output row)


def e4m3_value(q):
    """Value of FP8 E4M3 codes (OCP 8-bit float, the variant without infinities): sign bit, 4 exponent bits with
    bias 7, 3 mantissa bits; (-1)^s 2^(e-7) (1 + m/8) for e > 0, (-1)^s 2^-6 (m/8) for e = 0 (subnormals); the codes
    with e = 15 and m = 7 are NaN. Returned in fp64 (exact)."""
    q = np.asarray(q).astype(np.int64) & 0xFF
    sgn, e, m = q >> 7, (q >> 3) & 0xF, q & 7
    v = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return np.where(sgn == 1, -v, v)


def dequant_rows(q, scale):
    """Weights of an FP8 matrix [..., M, K] with one scale per output row [..., M]: W[m, k] = value(q[m, k]) *
    scale[m], exact in fp64."""
    return e4m3_value(q) * f64(scale)[..., None]


# --------------------------------------------------------------------------------------------------------------
# per-layer building blocks


def rmsnorm(x, g, eps):
    """RMSNorm over the last axis: x * (mean(x^2) + eps)^(-1/2) * g."""
    x = f64(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * f64(g)


def rope(x, pos, base):
    """1D rotary embedding [R] "Positional Embedding": x [..., n, heads, d] at absolute positions pos [n].

    Rotate-half pairing: element i pairs with i + d/2, angle pos * base^(-2i/d)."""
    x = f64(x)
    d = x.shape[-1]
    half = d // 2
    inv = base ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]      # [n, half]
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def block_visible(q_pos, k_pos, blk_len):
    """[R] "Block Diffusion Language Model (BDLM)": a query sees every key of its own block and of earlier
    blocks, none of later blocks. Blocks are [j*L, (j+1)*L) from position 0."""
    qb = np.asarray(q_pos, dtype=np.int64)[:, None] // blk_len
    kb = np.asarray(k_pos, dtype=np.int64)[None, :] // blk_len
    return kb <= qb


def attention(q, k, v, q_pos, k_pos, blk_len, scale=None):
    """Block-causal softmax attention for one batch row, two passes with an explicit mask.

    q [Lq, Hq, d], k/v [Nk, Hkv, d], q_pos [Lq], k_pos [Nk] -> o [Lq, Hq, d]."""
    q, k, v = f64(q), f64(k), f64(v)
    Lq, Hq, d = q.shape
    Hkv = k.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    vis = block_visible(q_pos, k_pos, blk_len)
    o = np.zeros_like(q)
    for h in range(Hq):
        g = h * Hkv // Hq
        s = (q[:, h, :] @ k[:, g, :].T) * scale
        s = np.where(vis, s, -np.inf)
        smax = s.max(axis=1, keepdims=True)
        p = np.exp(s - smax)
        p = p / p.sum(axis=1, keepdims=True)
        o[:, h, :] = p @ v[:, g, :]
    return o


def prefix_scores(k_prefix):
    """[R] "SPRINT" sparse prefix retention, key-norm term: l_i = mean over kv heads of ||K[h, i]||_2,
    mean-normalised over the prefix. k_prefix [Hkv, P, d] -> l~ [P]."""
    kk = f64(k_prefix)
    l = np.sqrt((kk * kk).sum(axis=-1)).mean(axis=0)
    return l / l.mean()


def prefix_importance(k_prefix, conf=None, alpha=1.0):
    """[R] "SPRINT": importance of prefix position i mixing the mean-normalised key norm l~_i with the top-1
    confidence c_i, alpha = 0.5 on the page (the formula itself was lost in extraction; the plain reading of the
    surrounding prose is the convex combination s_i = alpha l~_i + (1 - alpha) c_i). alpha = 1 (or no confidences)
    is the key-norm term alone. k_prefix [Hkv, P, d], conf [P] -> s [P]."""
    sc = prefix_scores(k_prefix)
    if conf is None or alpha == 1.0:
        return sc
    return alpha * sc + (1.0 - alpha) * f64(conf)


def prefix_retain(k_prefix, ratio, n_keep=None, conf=None, alpha=1.0, modality=None, n_keep_img=None):
    """Kept prefix positions, in position order. Without modality: the ceil(ratio * P) (or n_keep) positions of
    highest importance, ties -> lower position. With a modality mask ([M] "SPRINT 加速技术": modality-level keep
    ratios; [R] "SPRINT": image tokens are pruned more than text tokens): n_keep_img of the image positions
    (modality 1) and n_keep - n_keep_img of the text positions (modality 0), each the highest-importance ones of
    its modality, ties -> lower position.

    Returns (keep_pos [n_keep] int64, importance [P], margin) where margin is the smallest gap, within each
    modality, between the last kept and the first dropped position (inf when nothing is dropped)."""
    sc = prefix_importance(k_prefix, conf, alpha)
    P = sc.shape[0]
    if n_keep is None:
        n_keep = int(math.ceil(ratio * P))
    if modality is None:
        groups = [(list(range(P)), n_keep)]
    else:
        # a modality with fewer positions than its count keeps them all and the other keeps the rest (n_keep kept)
        mod = np.asarray(modality).astype(bool)
        img = [i for i in range(P) if mod[i]]
        txt = [i for i in range(P) if not mod[i]]
        ki = min(n_keep_img, len(img))
        kt = n_keep - ki
        if kt > len(txt):
            kt = len(txt)
            ki = n_keep - kt
        groups = [(img, ki), (txt, kt)]
    keep, margin = [], np.inf
    for pos, nk in groups:
        order = sorted(pos, key=lambda i: (-sc[i], i))
        keep += order[:nk]
        if 0 < nk < len(order):
            margin = min(margin, sc[order[nk - 1]] - sc[order[nk]])
        elif nk == 0 and order:
            margin = min(margin, np.inf)
    return np.array(sorted(keep), dtype=np.int64), sc, margin


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def route(h, w_router, bias, k, order=False):
    """[R] "MoE 백본" top-k router with the aux-loss-free bias of [R] "Load Balancing" used for selection only.

    h [T, H], w_router [E, H], bias [E] -> ids [T, k] (slots in biased-score order), gates [T, k],
    scores [T, E], margin [T]: the biased score of slot k-1 minus the best unchosen biased score (the gap that
    decides the chosen set), or with order=True the smallest gap between consecutive biased scores among the
    best k + 1 (the gaps that decide the set and the slot order)."""
    s = sigmoid(f64(h) @ f64(w_router).T)
    b = f64(bias)
    T, E = s.shape
    ids = np.zeros((T, k), dtype=np.int64)
    gates = np.zeros((T, k))
    margin = np.full(T, np.inf)
    for t in range(T):
        biased = s[t] + b
        order_t = sorted(range(E), key=lambda e: (-biased[e], e))
        ids[t] = order_t[:k]
        sel = s[t, ids[t]]
        gates[t] = sel / sel.sum()
        top = [biased[e] for e in order_t[:k + 1]]
        if order and len(top) > 1:
            margin[t] = min(top[j] - top[j + 1] for j in range(len(top) - 1))
        elif k < E:
            margin[t] = biased[order_t[k - 1]] - biased[order_t[k]]
    return ids, gates, s, margin


def silu(x):
    return x * sigmoid(x)


def swiglu_mlp(x, w_gu, w_down, dtype):
    """down(silu(gate x) * (up x)) for rows x [n, H]; w_gu [2I, H] = [gate; up], w_down [H, I].
    The activation is stored in ``dtype`` before the down projection."""
    x = f64(x)
    w_gu = f64(w_gu)
    I = w_gu.shape[0] // 2
    g = x @ w_gu[:I].T
    u = x @ w_gu[I:].T
    a = store(silu(g) * u, dtype)
    return a @ f64(w_down).T


def moe_delta(h, ids, gates, w_gu, w_down, w_gu_shared, w_down_shared, dtype):
    """MoE FFN output before the residual: shared(h_t) + sum_j gates[t, j] * expert_{ids[t, j]}(h_t).
    A plain per-token loop over the chosen experts (no permutation)."""
    h = f64(h)
    T = h.shape[0]
    out = np.zeros_like(h)
    for t in range(T):
        acc = np.zeros(h.shape[1])
        if w_gu_shared is not None:
            acc += swiglu_mlp(h[t:t + 1], w_gu_shared, w_down_shared, dtype)[0]
        for j in range(ids.shape[1]):
            e = int(ids[t, j])
            acc += gates[t, j] * swiglu_mlp(h[t:t + 1], w_gu[e], w_down[e], dtype)[0]
        out[t] = acc
    return out


# --------------------------------------------------------------------------------------------------------------
# confidence and unmasking


def cfg_combine(zc, zu, scale):
    """Classifier-free guidance z = z_u + s (z_c - z_u) (the guidance formula is not printed on the pages; this
    is the plain reading, s = cfg_scale), in fp64."""
    zc, zu = f64(zc), f64(zu)
    return zu + float(scale) * (zc - zu)


def cfg_fp32_error_bound(zc, zu, scale):
    """Largest rounding error, per row, of any evaluation of z_u + s (z_c - z_u) in float32 that rounds each of its
    three operations to nearest: with u = 2^-24, |fl(z) - z| <= u (2 |s (z_c - z_u)| + |z|) to first order (the
    subtraction's and the product's errors scale with s (z_c - z_u), the sum's with z); 1 % is added for the
    second-order terms. Comparison criteria use it to flag decisions that such rounding can flip."""
    zc, zu = f64(zc), f64(zu)
    d = float(scale) * (zc - zu)
    return 1.01 * 2.0 ** -24 * np.max(2.0 * np.abs(d) + np.abs(zu + d), axis=-1)


def cfg3_combine(zc, zi, zu, text_scale, image_scale):
    """Editing guidance with three rows per position (HF-mirror README, note under "SPRINT 加速技术": Editing CFG
    guides three ways through cfg_text_scale / cfg_image_scale; the formula is not printed on the pages, this is the
    plain reading): z = z_u + s_i (z_i - z_u) + s_t (z_c - z_i), with z_c the row conditioned on the instruction and
    the source image, z_i the row conditioned on the image only, z_u the unconditional row; s_t = cfg_text_scale,
    s_i = cfg_image_scale. In fp64."""
    zc, zi, zu = f64(zc), f64(zi), f64(zu)
    return zu + float(image_scale) * (zi - zu) + float(text_scale) * (zc - zi)


def cfg3_fp32_error_bound(zc, zi, zu, text_scale, image_scale):
    """Largest rounding error, per row, of the float32 evaluation a = z_u + s_i (z_i - z_u), z = a + s_t (z_c - z_i)
    with every operation rounded to nearest: with u = 2^-24, to first order |fl(z) - z| <= u (2 |m_i| + |a| +
    2 |m_t| + |z|), m_i = s_i (z_i - z_u), m_t = s_t (z_c - z_i) (each difference's error scales with its product);
    1 % is added for the second-order terms."""
    zc, zi, zu = f64(zc), f64(zi), f64(zu)
    mi = float(image_scale) * (zi - zu)
    mt = float(text_scale) * (zc - zi)
    a = zu + mi
    return 1.01 * 2.0 ** -24 * np.max(2.0 * np.abs(mi) + np.abs(a) + 2.0 * np.abs(mt) + np.abs(a + mt), axis=-1)


def confidence(z):
    """[R] "SPRINT": c = max_v softmax(z)_v, the candidate token is the lowest argmax.
    z [n, V] -> (cand [n] int64, c [n], lse [n], zmax [n])."""
    z = f64(z)
    zmax = z.max(axis=1)
    cand = z.argmax(axis=1)                  # numpy returns the first (lowest) index of the maximum
    lse = zmax + np.log(np.exp(z - zmax[:, None]).sum(axis=1))
    return cand.astype(np.int64), np.exp(zmax - lse), lse, zmax


SCORES = ("low_confidence", "top_k_margin", "neg_entropy")


def position_scores(z, score="low_confidence"):
    """Score by which [M] "SPRINT 加速技术" ranks the still-masked positions (its strategies low_confidence,
    top_k_margin, neg_entropy; the formulas are not on the pages, these are the plain readings of the names), from
    p = softmax(z) at temperature 1 over the scored vocabulary:
      low_confidence: p_(1), the largest probability (the c_i of [R] "SPRINT");
      top_k_margin:   p_(1) - p_(2), the two largest probabilities over distinct vocabulary entries (0 when the
                      largest logit occurs twice);
      neg_entropy:    sum_v p_v log p_v, the negated entropy (0 for a one-hot distribution, -log V for a uniform
                      one).
    z [n, V] -> score [n] (fp64)."""
    z = f64(z)
    zmax = z.max(axis=1, keepdims=True)
    e = np.exp(z - zmax)
    ssum = e.sum(axis=1)
    p = e / ssum[:, None]
    if score == "low_confidence":
        return p.max(axis=1)
    if score == "top_k_margin":
        top2 = np.sort(p, axis=1)[:, -2:] if p.shape[1] > 1 else np.concatenate([np.zeros_like(p), p], axis=1)
        return top2[:, 1] - top2[:, 0]
    if score == "neg_entropy":
        # sum_v p_v log p_v with log p_v = (z_v - zmax) - log(sum); terms with p_v = 0 contribute 0
        logp = (z - zmax) - np.log(ssum)[:, None]
        return (p * logp).sum(axis=1)
    raise ValueError(score)


def unmask_count(m, t, T_s, mode, tau=None, k_max=None, conf_masked=None):
    """Positions to unmask at step t (0-based) of T_s with m still masked.

    fixed ([M] "SPRINT 加速技术", [R] standard schedule): ceil(m / (T_s - t)).
    threshold ([R] "SPRINT" non-uniform unmasking, [M] batch acceptance): every c > tau, capped at k_max, and
    never fewer than ceil(m / (T_s - t)); never more than m."""
    if m == 0:
        return 0
    floor_k = -(-m // (T_s - t))
    if mode == 0:
        return min(m, floor_k)
    above = int(np.sum(np.asarray(conf_masked) > tau))
    return min(m, max(floor_k, min(k_max, above)))


def select_positions(conf_row, masked_row, k):
    """The k masked positions of one block row with the highest confidence, ties -> lower position.
    Returns (chosen positions in rank order, margin between rank k-1 and rank k, or inf)."""
    pos = [i for i in range(len(masked_row)) if masked_row[i]]
    order = sorted(pos, key=lambda i: (-conf_row[i], i))
    margin = conf_row[order[k - 1]] - conf_row[order[k]] if 0 < k < len(order) else np.inf
    return order[:k], margin


def unmask(z_rows, row_pos, tokens, mask, t, T_s, mode=0, tau=0.9, k_max=8, vocab_offset=0,
           z_uncond=None, cfg_scale=1.0, score="low_confidence", z_image=None, cfg_image_scale=1.0):
    """One unmasking step over a batch of block rows.

    z_rows [n, V]: logits of the still-masked positions, row r belongs to flat position row_pos[r] = b*L + i of
    the conditional rows. With ``z_uncond`` given, the rows are combined by CFG first (fp64), and the selection
    is written to both halves of the batch (rows b and b + B/2). With ``z_image`` given too (editing guidance), the
    three rows of a position are combined by cfg3_combine and the selection is written to the three thirds of the
    batch (rows b, b + B/3, b + 2B/3).

    Near-tie flags (decisions a correct implementation may take either way): a confidence margin below 1e-6
    relative between the last chosen and the first unchosen position (tie_rank), a confidence within 1e-6 of tau
    (tie_tau). A library that evaluates the guidance in float32 perturbs each guided logit by up to
    cfg_fp32_error_bound (z_err per row); the bands then widen by that amount: a candidate whose top-2 guided-logit
    gap is at most 2 z_err (tie_cand), and confidences, which move by a relative 2 z_err at most (conf_rtol).
    score: the strategy that ranks the positions (position_scores); the threshold acceptance always counts the
    positions whose largest probability exceeds tau ([M] "SPRINT 加速技术": tokens whose probability exceeds the
    threshold are accepted).
    Returns dict(tokens, mask, sel [Bl, k], nsel [Bl], conf [Bl, L] (largest probability), rank [Bl, L] (ranking
    score), cand [Bl, L], tie_rank [Bl], tie_tau [Bl], tie_cand [Bl, L], conf_rtol [Bl, L]) where Bl is the number
    of logical rows."""
    tokens = np.array(tokens, dtype=np.int64, copy=True)
    mask = np.array(mask, dtype=np.int64, copy=True)
    B, L = mask.shape
    groups = 1 if z_uncond is None else (3 if z_image is not None else 2)
    Bl = B // groups
    if z_image is not None:
        z = cfg3_combine(z_rows, z_image, z_uncond, cfg_scale, cfg_image_scale)
        z_err = cfg3_fp32_error_bound(z_rows, z_image, z_uncond, cfg_scale, cfg_image_scale)
    elif z_uncond is not None:
        z = cfg_combine(z_rows, z_uncond, cfg_scale)
        z_err = cfg_fp32_error_bound(z_rows, z_uncond, cfg_scale)
    else:
        z = f64(z_rows)
        z_err = np.zeros(z.shape[0])
    cand_r, conf_r, _, _ = confidence(z)
    rank_r = conf_r if score == "low_confidence" else position_scores(z, score)
    if z.shape[1] > 1:
        top2 = np.sort(z, axis=1)[:, -2:]
        gap_r = top2[:, 1] - top2[:, 0]
    else:
        gap_r = np.full(z.shape[0], np.inf)
    conf = np.zeros((Bl, L))
    rank = np.zeros((Bl, L))
    cand = np.full((Bl, L), -1, dtype=np.int64)
    tie_cand = np.zeros((Bl, L), dtype=bool)
    conf_rtol = np.full((Bl, L), 1e-6)
    for r, p in enumerate(row_pos):
        b, i = divmod(int(p), L)
        conf[b, i] = conf_r[r]
        rank[b, i] = rank_r[r]
        cand[b, i] = cand_r[r] + vocab_offset
        tie_cand[b, i] = z_err[r] > 0 and gap_r[r] <= 2.0 * z_err[r]
        conf_rtol[b, i] = 1e-6 + 2.0 * z_err[r]
    sel, nsel = [], np.zeros(Bl, dtype=np.int64)
    tie_rank = np.zeros(Bl, dtype=bool)
    tie_tau = np.zeros(Bl, dtype=bool)
    for b in range(Bl):
        masked = mask[b].astype(bool)
        m = int(masked.sum())
        cm = conf[b][masked]
        kt = unmask_count(m, t, T_s, mode, tau, k_max, cm)
        chosen, margin = select_positions(rank[b], masked, kt)
        band = 2.0 * float(conf_rtol[b].max())
        tie_rank[b] = margin < band * max(np.abs(rank[b][masked]).max() if m else 0.0, 1e-30)
        if mode == 1 and m:
            tie_tau[b] = bool(np.any(np.abs(cm - tau) < 1e-6 + conf_rtol[b][masked] * cm))
        for i in chosen:
            tokens[b, i] = cand[b, i]
            mask[b, i] = 0
            for grp in range(1, groups):   # the guidance rows of the same position take the same token
                tokens[b + grp * Bl, i] = cand[b, i]
                mask[b + grp * Bl, i] = 0
        sel.append(chosen)
        nsel[b] = kt
    return dict(tokens=tokens, mask=mask, sel=sel, nsel=nsel, conf=conf, rank=rank, cand=cand,
                tie_rank=tie_rank, tie_tau=tie_tau, tie_cand=tie_cand, conf_rtol=conf_rtol)


# --------------------------------------------------------------------------------------------------------------
# the denoising pass


def _layer_kv(h_rows, lw, w, pos):
    """q/k/v of rows h_rows [n, H] at positions pos: GEMM, RoPE on q and k, storage rounding."""
    qkv = f64(h_rows) @ f64(lw["w_qkv"]).T
    Hq, Hkv, d = w.Hq, w.Hkv, w.d
    n = qkv.shape[0]
    q = qkv[:, : Hq * d].reshape(n, Hq, d)
    k = qkv[:, Hq * d: (Hq + Hkv) * d].reshape(n, Hkv, d)
    v = qkv[:, (Hq + Hkv) * d:].reshape(n, Hkv, d)
    q = store(rope(q, pos, w.rope_base), w.dtype)
    k = store(rope(k, pos, w.rope_base), w.dtype)
    v = store(v, w.dtype)
    return q, k, v


def forward_block(w, weights, caches, tokens, mask, keep=None, want_logits=True, skip_last_ffn=False):
    """The backbone over one block for every batch row.

    w: workload (dims, dtype, eps, rope_base, blk len L, prefix length P); weights: dict from the synthetic
    generator (torch or numpy arrays); caches: per layer (K, V) [B, Hkv, >=P, d]; tokens/mask [B, L].
    keep: per layer, per row, array of kept prefix positions (SPRINT) or None for the full prefix.
    Returns dict(x [B, L, H] final hidden before the final norm, block_k / block_v per layer [B, L, Hkv, d],
    route per layer (ids, gates, margin), logits [n_m, vlen] for the masked rows, row_pos [n_m])."""
    B, L, P, H = w.B, w.L, w.P, w.H
    dt = w.dtype
    tok = np.where(np.asarray(mask).astype(bool), w.mask_id, np.asarray(tokens))
    emb = weights["embed"]
    x = np.stack([f64(emb[int(i)]) for i in tok.reshape(-1)]).reshape(B * L, H)     # exact copy of the rows
    pos = np.arange(P, P + L)
    out = dict(block_k=[], block_v=[], route=[])
    n_layers = len(weights["layers"])
    for li, lw in enumerate(weights["layers"]):
        kc, vc = f64(caches[li][0]), f64(caches[li][1])
        h = store(rmsnorm(x, lw["attn_norm"], w.eps), dt)
        o = np.zeros((B, L, w.Hq, w.d))
        bk = np.zeros((B, L, w.Hkv, w.d))
        bv = np.zeros((B, L, w.Hkv, w.d))
        for b in range(B):
            q, k, v = _layer_kv(h[b * L:(b + 1) * L], lw, w, pos)
            bk[b], bv[b] = k, v
            kp = np.arange(P) if keep is None else np.asarray(keep[li][b])
            keys = np.concatenate([kc[b][:, kp, :].transpose(1, 0, 2), k], axis=0)
            vals = np.concatenate([vc[b][:, kp, :].transpose(1, 0, 2), v], axis=0)
            kpos = np.concatenate([kp, pos])
            o[b] = store(attention(q, keys, vals, pos, kpos, L), dt)
        out["block_k"].append(bk)
        out["block_v"].append(bv)
        x = store(x + o.reshape(B * L, -1) @ f64(lw["w_o"]).T, dt)
        if skip_last_ffn and li == n_layers - 1:
            out["route"].append(None)
            break
        h2 = store(rmsnorm(x, lw["ffn_norm"], w.eps), dt)
        ids, gates, _, margin = route(h2, lw["w_router"], lw["router_bias"], w.k)
        out["route"].append((ids, gates, margin))
        delta = moe_delta(h2, ids, gates, lw["w_gu"], lw["w_down"], lw["w_gu_shared"], lw["w_down_shared"], dt)
        x = store(x + delta, dt)
    out["x"] = x.reshape(B, L, H)
    if want_logits:
        xf = store(rmsnorm(x, weights["final_norm"], w.eps), dt)
        groups = 1 + w.cfg   # cfg 1: (cond, uncond) halves; cfg 2 (editing): (cond, image-only, uncond) thirds
        Bl = B // groups
        row_pos = np.nonzero(np.asarray(mask)[:Bl].reshape(-1))[0]
        rows = [p + grp * Bl * L for grp in range(groups) for p in row_pos]
        wl = f64(weights["w_lm"][w.vocab_offset: w.vocab_offset + w.vlen])
        out["logits"] = store(xf[rows] @ wl.T, dt)
        out["row_pos"] = row_pos
    return out


def denoise_step(w, weights, caches, tokens, mask, t, keep=None):
    """One denoising pass at step t: backbone, LM head over the masked rows, confidence, unmasking."""
    f = forward_block(w, weights, caches, tokens, mask, keep=keep)
    n = len(f["row_pos"])
    z = f["logits"]
    zi = None
    if w.cfg == 2:
        zc, zi, zu = z[:n], z[n:2 * n], z[2 * n:]
    elif w.cfg:
        zc, zu = z[:n], z[n:]
    else:
        zc, zu = z, None
    u = unmask(zc, f["row_pos"], tokens, mask, t, w.T_s, w.mode, w.tau, w.k_max, w.vocab_offset,
               z_uncond=zu, cfg_scale=w.cfg_scale, score=SCORES[getattr(w, "score", 0)], z_image=zi,
               cfg_image_scale=getattr(w, "cfg_image_scale", 1.0))
    u["forward"] = f
    return u


def commit_block(w, weights, caches, tokens, keep=None):
    """Pass over the finished block's clean tokens ([R] BDLM: earlier blocks are always clean context): each
    layer's block K/V [B, L, Hkv, d] for cache rows [P, P + L). The last layer's FFN and the LM head have no
    consumer and are skipped."""
    mask = np.zeros_like(np.asarray(tokens))
    f = forward_block(w, weights, caches, tokens, mask, keep=keep, want_logits=False, skip_last_ffn=True)
    return f["block_k"], f["block_v"]


def sprint_keep(w, caches, conf=None, modality=None):
    """SPRINT selection at the first step of a block: per layer, per row, kept prefix positions (conf [B, P] and
    modality [P] as in prefix_retain, with the workload's alpha and keep counts)."""
    keep = []
    alpha = getattr(w, "sprint_alpha", 1.0)
    n_img = getattr(w, "n_keep_img", None)
    for li in range(len(caches)):
        kc = f64(caches[li][0])
        keep.append([prefix_retain(kc[b][:, : w.P, :], w.keep_ratio, n_keep=w.n_keep,
                                   conf=None if conf is None else conf[b][: w.P], alpha=alpha,
                                   modality=None if modality is None else modality[: w.P], n_keep_img=n_img)[0]
                     for b in range(w.B)])
    return keep
