"""Helpers shared by the GPU parity tests (comparison criteria and small input builders)."""
import numpy as np
import torch

# float tolerances of the parity bar: bf16 storage -> max-abs <= 2e-2 and relative L2 <= 5e-3; fp32 -> 1e-4.
# Per element the bf16 bound is max(2e-2 * scale, ulps * ulp(value)): both sides round results that differ by
# ~1e-6 relative to bf16, so each rounding may land on either neighbour of a boundary (one ulp = 2^-7 relative
# at most); a value that went through two such roundings (the residual stream: after attention and after the
# MoE FFN) may be two ulps apart. `scale` carries a known amplification of upstream one-ulp differences (logits:
# the LM-head weight scale relative to 0.02).
TOL = {"bf16": (2e-2, 5e-3), "f32": (1e-4, 1e-4)}


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(got, want, dtype, what="", ulps=1, scale=1.0):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    abs_tol, rel_tol = TOL[dtype]
    err = np.abs(got - want)
    max_abs = float(err.max()) if err.size else 0.0
    rel_l2 = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    if dtype == "f32":
        # fp32: 1e-4 absolute or relative per element
        bad = err > abs_tol * np.maximum(1.0, np.abs(want))
        assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond 1e-4 (max abs {max_abs:.3g})"
    else:
        bound = np.maximum(abs_tol * scale, ulps * np.abs(want) * 2.0 ** -7)
        bad = err > bound
        assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond max(2e-2, one bf16 ulp); "
                               f"max-abs {max_abs:.4g}")
        assert rel_l2 <= rel_tol, f"{what}: rel-L2 {rel_l2:.4g} > {rel_tol}"
    return max_abs, rel_l2


def assignment_tables(ids, E):
    """counts, offsets, perm, inv of the (token, slot) assignments grouped by expert, stable in token order."""
    T, k = ids.shape
    flat = ids.reshape(-1)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(len(perm), dtype=np.int32)
    return counts, offsets, perm, inv


def random_assignments(T, E, k, seed):
    g = np.random.default_rng(seed)
    ids = np.stack([g.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    gates = g.uniform(0.1, 1.0, (T, k)).astype(np.float32)
    gates = (gates / gates.sum(1, keepdims=True)).astype(np.float32)
    return ids, gates


# Router near-tie band: the chosen expert ids (in slot order) must equal the oracle's wherever every gap between
# consecutive biased scores among the oracle's best k + 1 is at least this (the criterion of the parity bar).
ROUTE_TIE = 1e-6


def same_routing(g_ids, g_gates, o_ids, o_gates, rows, rtol, atol):
    """On `rows`, the library's expert ids equal the oracle's slot by slot, and the gates agree."""
    g_ids, o_ids = np.asarray(g_ids)[rows], np.asarray(o_ids)[rows]
    bad = np.nonzero(~np.all(g_ids == o_ids, axis=1))[0]
    assert len(bad) == 0, f"routed expert ids differ away from near-ties at {len(bad)} tokens, e.g. " \
        f"{g_ids[bad[0]].tolist()} vs {o_ids[bad[0]].tolist()}" if len(bad) else ""
    assert np.allclose(np.asarray(g_gates)[rows], np.asarray(o_gates)[rows], rtol=rtol, atol=atol)


def check_unmask(u, conf, nsel, sel, tokens, mask, Bl, cfg):
    """Library unmask outputs (numpy) against the oracle's dict u: confidences within u["conf_rtol"] at masked
    positions; for every logical row whose decision is not a near-tie (u["tie_rank"], u["tie_tau"]) the count,
    the chosen positions in rank order and the mask exactly, and the written tokens exactly except where the
    candidate itself is a near-tie (u["tie_cand"]); with cfg (1 or 2) the guidance rows b + g * Bl too."""
    m_ = u["conf"] > 0
    err = np.abs(conf.astype(np.float64) - u["conf"])
    assert np.all(err[m_] <= u["conf_rtol"][m_] * u["conf"][m_] + 1e-12), "confidences differ"
    for b in range(Bl):
        if u["tie_rank"][b] or u["tie_tau"][b]:
            continue
        assert nsel[b] == u["nsel"][b], f"row {b}: count"
        assert list(sel[b][: u["nsel"][b]]) == list(u["sel"][b]), f"row {b}: chosen positions"
        assert np.array_equal(mask[b], u["mask"][b]), f"row {b}: mask"
        ok = ~u["tie_cand"][b]
        assert np.array_equal(tokens[b][ok], u["tokens"][b][ok]), f"row {b}: tokens"
        for g in range(1, 1 + int(cfg)):
            assert np.array_equal(mask[b + g * Bl], u["mask"][b + g * Bl]), f"row {b} group {g}: mask"
            assert np.array_equal(tokens[b + g * Bl][ok], u["tokens"][b + g * Bl][ok]), f"row {b} group {g}: tokens"
