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


# Router near-tie band. The library scores experts in fp32 (tensor-core accumulation over H), within 2e-6 of the
# fp64 oracle's sigmoid scores (asserted by the router tests); two experts whose exact biased scores differ by less
# than twice that can swap, so a selection whose oracle margin is below ROUTE_TIE is a near-tie.
ROUTE_TIE = 4e-6


def same_selection(g_ids, g_gates, o_ids, o_gates, rows, rtol, atol):
    """The chosen expert sets agree on `rows`, and every chosen expert's gate agrees. The slot order is the
    library's fp32 score order, which may differ from the exact order only between experts whose scores lie within
    the fp32 error of each other; it decides nothing but the order of the combine's sum."""
    g_ids, o_ids = np.asarray(g_ids)[rows], np.asarray(o_ids)[rows]
    gs, os_ = np.argsort(g_ids, axis=1), np.argsort(o_ids, axis=1)
    assert np.array_equal(np.take_along_axis(g_ids, gs, 1), np.take_along_axis(o_ids, os_, 1)), \
        "routed expert sets differ away from near-ties"
    assert np.allclose(np.take_along_axis(np.asarray(g_gates)[rows], gs, 1),
                       np.take_along_axis(np.asarray(o_gates)[rows], os_, 1), rtol=rtol, atol=atol)


def slot_order_valid(ids, scores, bias, guard=None):
    """Slots are in non-increasing biased-score order up to the fp32 error band."""
    guard = ROUTE_TIE if guard is None else guard
    v = np.take_along_axis(np.asarray(scores, dtype=np.float64), np.asarray(ids, dtype=np.int64), 1) + \
        np.asarray(bias, dtype=np.float64)[np.asarray(ids, dtype=np.int64)]
    assert np.all(np.diff(v, axis=1) <= guard), "slots out of biased-score order"

