"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test names the passage it rests on. None of them compares the oracle with
itself: the references are closed-form counts, a library attention routine
(torch scaled_dot_product_attention / logsumexp / autograd in float64),
finite differences, exact special cases and exact invariants.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import reference_np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

CASES_SMALL = [
    # kind, mode, T, l, c
    ("strided", "split", 48, 5, 1),
    ("strided", "merged", 48, 5, 1),
    ("strided", "split", 64, 8, 1),
    ("strided", "merged", 64, 16, 1),
    ("fixed", "split", 48, 8, 2),
    ("fixed", "merged", 48, 8, 2),
    ("fixed", "split", 64, 16, 4),
    ("fixed", "merged", 64, 16, 1),
    ("fixed", "merged", 40, 6, 3),
    ("dense", "merged", 33, 1, 1),
]


# ---- index sets: exact counts ---------------------------------------------

def strided_counts(i, l):
    """|A1|, |A2|, |A1 u A2| from the set definitions (Sparse Transformer,
    llm-arch-kb section 2, Pattern A: window of the last l keys, every l-th
    key back)."""
    a1 = min(i, l) + 1
    a2 = i // l + 1
    union = i + 1 if i < l else l + i // l
    return a1, a2, union


def fixed_counts(i, l, c):
    """Same for Pattern B: own block, last c positions of every block."""
    r = i % l
    a1 = r + 1
    a2 = c * (i // l) + max(0, r - (l - c) + 1)
    union = r + 1 + c * (i // l)
    return a1, a2, union


@pytest.mark.parametrize("T,l", [(50, 7), (64, 8), (100, 10), (256, 16), (300, 300), (90, 200)])
def test_strided_row_counts_closed_form(orc, T, l):
    for i in range(T):
        a1, a2, un = strided_counts(i, l)
        assert len(orc.row_set("strided", "split", l, 1, 0, i)) == a1
        assert len(orc.row_set("strided", "split", l, 1, 1, i)) == a2
        assert len(orc.row_set("strided", "merged", l, 1, 0, i)) == un
        if i >= l:
            # the pages' approximation |A1|+|A2|-1 ~ l + ceil(i/l) (llm-arch-kb section 2)
            assert abs(un - (l + math.ceil(i / l))) <= 1


@pytest.mark.parametrize("T,l,c", [(64, 8, 2), (100, 10, 3), (256, 16, 4), (128, 32, 32), (70, 9, 1)])
def test_fixed_row_counts_closed_form(orc, T, l, c):
    for i in range(T):
        a1, a2, un = fixed_counts(i, l, c)
        assert len(orc.row_set("fixed", "split", l, c, 0, i)) == a1
        assert len(orc.row_set("fixed", "split", l, c, 1, i)) == a2
        s = orc.row_set("fixed", "merged", l, c, 0, i)
        assert len(s) == un
        # the pages' bound |B1|+|B2| <= l + c ceil(i/l) (llm-arch-kb section 2, Pattern B)
        assert un <= l + c * math.ceil(i / l)


def test_sets_are_causal_sorted_and_head_parity(orc):
    T, l, c = 80, 8, 3
    for kind in ("strided", "fixed"):
        for i in range(T):
            even = orc.row_set(kind, "split", l, c, 0, i)
            even2 = orc.row_set(kind, "split", l, c, 6, i)
            odd = orc.row_set(kind, "split", l, c, 1, i)
            odd2 = orc.row_set(kind, "split", l, c, 5, i)
            assert np.array_equal(even, even2) and np.array_equal(odd, odd2)
            for s in (even, odd, orc.row_set(kind, "merged", l, c, 3, i)):
                assert np.all(np.diff(s) > 0)
                assert s.size == 0 or (s[0] >= 0 and s[-1] <= i)
            merged = orc.row_set(kind, "merged", l, c, 1, i)
            assert np.array_equal(merged, np.union1d(even, odd))


def test_sets_match_membership_brute_force(orc):
    """Constructive enumeration == pairwise membership test of the definitions."""
    for kind, mode, T, l, c in CASES_SMALL:
        for h in (0, 1):
            m = reference_np.mask(kind, mode, T, l, c, h)
            for i in range(T):
                s = orc.row_set(kind, mode, l, c, h, i)
                assert np.array_equal(s, np.nonzero(m[i])[0]), (kind, mode, h, i)


def test_cost_model_total(orc):
    """Sum_i (l + i/l) ~ T l + T^2/(2l) for the strided pattern (llm-arch-kb
    section 2); within 0.5% at T = 65536, l = 256 = sqrt(T)."""
    T, l = 65536, 256
    n = orc.nnz("strided", "merged", T, l, 1, 0)
    approx = T * l + T * T / (2 * l)
    assert abs(n - approx) / approx < 0.005


def test_nnz_golden(orc):
    """Per-workload live-pair totals, derived by closed-form summation of the
    exact row counts (see the fixture's note)."""
    with open(os.path.join(GOLDEN, "nnz.json")) as f:
        gold = json.load(f)
    for name, g in gold["workloads"].items():
        kind, mode, T, l, c = g["kind"], g["mode"], g["T"], g["l"], g["c"]
        if mode == "split":
            n0 = orc.nnz(kind, mode, T, l, c, 0)
            n1 = orc.nnz(kind, mode, T, l, c, 1)
            assert n0 == g["per_head_even"], name
            assert n1 == g["per_head_odd"], name
            H = g["H"]
            tot = g["B"] * ((H + 1) // 2 * n0 + H // 2 * n1)
        else:
            n0 = orc.nnz(kind, mode, T, l, c, 0)
            assert n0 == g["per_head"], name
            tot = g["B"] * g["H"] * n0
        assert tot == g["total"], name
        # and the closed forms summed here
        if kind == "strided":
            f = strided_counts
            cs = [f(i, l) for i in range(T)]
        else:
            cs = [fixed_counts(i, l, c) for i in range(T)]
        if mode == "split":
            assert sum(x[0] for x in cs) == n0 and sum(x[1] for x in cs) == n1
        else:
            assert sum(x[2] for x in cs) == n0


# ---- two-hop reachability --------------------------------------------------

@pytest.mark.parametrize("kind,T,l,c", [("strided", 120, 7, 1), ("strided", 200, 14, 1),
                                        ("fixed", 120, 8, 1), ("fixed", 200, 14, 3)])
def test_two_hop_reachability(orc, kind, T, l, c):
    """Every earlier k is reachable from i in at most two hops of the merged
    pattern (llm-arch-kb section 2, "Two-hop reachability"); in split mode,
    through the A2 head then the A1 head (nlp-lineage milestone, The idea)."""
    merged = [set(orc.row_set(kind, "merged", l, c, 0, i).tolist()) for i in range(T)]
    a1 = [set(orc.row_set(kind, "split", l, c, 0, i).tolist()) for i in range(T)]
    a2 = [set(orc.row_set(kind, "split", l, c, 1, i).tolist()) for i in range(T)]
    for i in range(T):
        reach_m = set(merged[i])
        for j in merged[i]:
            reach_m |= merged[j]
        reach_s = set(a1[i])
        for j in a2[i]:
            reach_s |= a1[j]
        for k in range(i):
            assert k in reach_m, (kind, i, k)
            assert k in reach_s, (kind, i, k)


# ---- attention arithmetic vs a library routine ------------------------------

def _inputs(B, H, T, d, seed):
    g = torch.Generator().manual_seed(seed)
    q, k, v, do = (torch.randn(B, H, T, d, generator=g) for _ in range(4))
    return q, k, v, do


@pytest.mark.parametrize("case", CASES_SMALL)
def test_forward_equals_dense_masked_sdpa(orc, case):
    """Sparse attention == dense attention with excluded logits at -inf
    (llm-arch-kb section 2, "Sparse attention as an unnormalized form"),
    computed by torch's scaled_dot_product_attention in float64."""
    kind, mode, T, l, c = case
    B, H, d = 1, 3, 8
    q, k, v, _ = _inputs(B, H, T, d, 1)
    o, lse = orc.forward(kind, mode, q.numpy(), k.numpy(), v.numpy(), l, c)
    for h in range(H):
        m = torch.from_numpy(reference_np.mask(kind, mode, T, l, c, h))
        q64, k64, v64 = (x[0, h].double() for x in (q, k, v))
        ref = F.scaled_dot_product_attention(q64[None], k64[None], v64[None], attn_mask=m[None])[0]
        s = (q64 @ k64.T) / math.sqrt(d)
        ref_lse = torch.logsumexp(s.masked_fill(~m, -math.inf), dim=-1)
        empty = ~m.any(dim=1)
        ok = ~empty
        np.testing.assert_allclose(o[0, h][ok.numpy()], ref[ok].numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, h][ok.numpy()], ref_lse[ok].numpy(), rtol=0, atol=1e-12)
        # empty rows: O = 0 and LSE = -inf (no keys contribute mass)
        assert np.all(o[0, h][empty.numpy()] == 0.0)
        assert np.all(np.isneginf(lse[0, h][empty.numpy()]))


def test_empty_rows_exist_where_expected(orc):
    """Fixed split, A2 head: rows i < l-c of block 0 see no summary key."""
    T, l, c = 64, 16, 4
    for i in range(T):
        s = orc.row_set("fixed", "split", l, c, 1, i)
        assert (s.size == 0) == (i < l - c)


@pytest.mark.parametrize("case", CASES_SMALL[:6])
def test_backward_equals_autograd_on_masked_sdpa(orc, case):
    kind, mode, T, l, c = case
    B, H, d = 1, 2, 8
    q, k, v, do = _inputs(B, H, T, d, 2)
    dq, dk, dv = orc.backward(kind, mode, q.numpy(), k.numpy(), v.numpy(), do.numpy(), l, c)
    for h in range(H):
        m = torch.from_numpy(reference_np.mask(kind, mode, T, l, c, h))
        empty = ~m.any(dim=1)
        m2 = m.clone()
        m2[empty, 0] = True  # keep SDPA finite; those rows get dO = 0 below
        q64, k64, v64 = (x[0, h].double().clone().requires_grad_(True) for x in (q, k, v))
        do64 = do[0, h].double().clone()
        do64[empty] = 0.0
        out = F.scaled_dot_product_attention(q64[None], k64[None], v64[None], attn_mask=m2[None])[0]
        (out * do64).sum().backward()
        np.testing.assert_allclose(dq[0, h][~empty.numpy()], q64.grad[~empty].numpy(), atol=1e-11)
        if not empty.any():
            np.testing.assert_allclose(dk[0, h], k64.grad.numpy(), atol=1e-11)
            np.testing.assert_allclose(dv[0, h], v64.grad.numpy(), atol=1e-11)


def test_backward_finite_differences(orc):
    """Central differences of L = sum(O * dO) in float64, T = 24."""
    rng = np.random.default_rng(5)
    for kind, mode, l, c in [("strided", "merged", 5, 1), ("fixed", "split", 6, 2),
                             ("fixed", "merged", 6, 2), ("strided", "split", 4, 1)]:
        B, H, T, d = 1, 2, 24, 4
        # float32 inputs that are exact dyadic rationals keep perturbations exact
        q, k, v, do = (np.round(rng.standard_normal((B, H, T, d)) * 64) / 64 for _ in range(4))
        q, k, v, do = (x.astype(np.float32) for x in (q, k, v, do))
        dq, dk, dv = orc.backward(kind, mode, q, k, v, do, l, c)
        eps = 2.0 ** -10

        def loss(qq, kk, vv):
            o, _ = orc.forward(kind, mode, qq, kk, vv, l, c)
            return float((o * do.astype(np.float64)).sum())

        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            idx = [tuple(rng.integers(0, s) for s in x.shape) for _ in range(12)]
            for ix in idx:
                xp = x.copy(); xp[ix] += eps
                xm = x.copy(); xm[ix] -= eps
                args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
                args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
                num = (loss(*args_p) - loss(*args_m)) / (2 * eps)
                assert abs(num - g[ix]) < 2e-5 * max(1.0, abs(g[ix])), (kind, mode, name, ix)


def test_gradient_invariants(orc):
    """Exact: sum_j dK_j = 0 per head (softmax is invariant to k_j -> k_j + u),
    and sum_j dV_j = sum over non-empty rows of dO_i (rows of P sum to 1)."""
    B, H, T, d = 1, 4, 96, 8
    q, k, v, do = _inputs(B, H, T, d, 3)
    for kind, mode, l, c in [("fixed", "split", 16, 4), ("strided", "merged", 12, 1),
                             ("fixed", "merged", 8, 3)]:
        dq, dk, dv = orc.backward(kind, mode, q.numpy(), k.numpy(), v.numpy(), do.numpy(), l, c)
        for h in range(H):
            assert np.abs(dk[0, h].sum(axis=0)).max() < 1e-10
            nonempty = np.array([orc.row_set(kind, mode, l, c, h, i).size > 0 for i in range(T)])
            ref = do[0, h].double().numpy()[nonempty].sum(axis=0)
            np.testing.assert_allclose(dv[0, h].sum(axis=0), ref, atol=1e-10)


# ---- closed-form outputs and special cases -----------------------------------

def test_zero_queries_give_uniform_average(orc):
    """Q = 0 makes every allowed logit equal: O_i is the mean of v_j over S_i
    and LSE_i = ln |S_i|."""
    B, H, T, d = 1, 2, 70, 6
    _, k, v, _ = _inputs(B, H, T, d, 4)
    q = torch.zeros(B, H, T, d)
    for kind, mode, l, c in [("strided", "split", 9, 1), ("fixed", "merged", 10, 3),
                             ("fixed", "split", 10, 3)]:
        o, lse = orc.forward(kind, mode, q.numpy(), k.numpy(), v.numpy(), l, c)
        for h in range(H):
            for i in range(T):
                s = orc.row_set(kind, mode, l, c, h, i)
                if s.size == 0:
                    continue
                ref = v[0, h, s].double().mean(dim=0).numpy()
                np.testing.assert_allclose(o[0, h, i], ref, atol=1e-14)
                assert abs(lse[0, h, i] - math.log(s.size)) < 1e-14


def test_constant_values_pass_through(orc):
    B, H, T, d = 1, 2, 50, 5
    q, k, _, _ = _inputs(B, H, T, d, 6)
    u = torch.arange(d, dtype=torch.float32) * 0.25 - 0.5
    v = u.expand(B, H, T, d).contiguous()
    o, _ = orc.forward("fixed", "merged", q.numpy(), k.numpy(), v.numpy(), 7, 2)
    np.testing.assert_allclose(o, np.broadcast_to(u.double().numpy(), o.shape), atol=1e-14)


def test_l_at_least_T_reduces(orc):
    """l >= T: merged and A1 heads become full causal attention; the strided A2
    head sees only itself (O_i = v_i, LSE_i = s_ii); the fixed A2 head sees
    {j : l-c <= j <= i}."""
    B, H, T, d = 1, 2, 40, 4
    q, k, v, _ = _inputs(B, H, T, d, 7)
    od, ld = orc.forward("dense", "merged", q.numpy(), k.numpy(), v.numpy(), 1, 1)
    for kind, mode, l, c in [("strided", "merged", 40, 1), ("strided", "split", 64, 1),
                             ("fixed", "merged", 40, 4), ("fixed", "split", 50, 4)]:
        o, lse = orc.forward(kind, mode, q.numpy(), k.numpy(), v.numpy(), l, c)
        heads = [0, 1] if mode == "merged" else [0]
        for h in heads:
            np.testing.assert_allclose(o[0, h], od[0, h], atol=1e-13)
            np.testing.assert_allclose(lse[0, h], ld[0, h], atol=1e-13)
    o, lse = orc.forward("strided", "split", q.numpy(), k.numpy(), v.numpy(), 64, 1)
    np.testing.assert_allclose(o[0, 1], v[0, 1].double().numpy(), atol=1e-14)
    sii = (q[0, 1].double() * k[0, 1].double()).sum(-1).numpy() / math.sqrt(d)
    np.testing.assert_allclose(lse[0, 1], sii, atol=1e-14)
    l, c = 50, 15
    for i in range(T):
        s = orc.row_set("fixed", "split", l, c, 1, i)
        assert np.array_equal(s, np.arange(l - c, i + 1))


# ---- the two restatements agree; sampled rows agree with full passes -------

@pytest.mark.parametrize("case", CASES_SMALL)
def test_cpp_matches_numpy_restatement(orc, case):
    kind, mode, T, l, c = case
    q, k, v, do = _inputs(1, 2, T, 8, 8)
    o, lse = orc.forward(kind, mode, q.numpy(), k.numpy(), v.numpy(), l, c)
    o2, lse2 = reference_np.forward(kind, mode, q.numpy(), k.numpy(), v.numpy(), l, c)
    np.testing.assert_allclose(o, o2, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lse2))
    fin = np.isfinite(lse)
    np.testing.assert_allclose(lse[fin], lse2[fin], atol=1e-12)
    g = orc.backward(kind, mode, q.numpy(), k.numpy(), v.numpy(), do.numpy(), l, c)
    g2 = reference_np.backward(kind, mode, q.numpy(), k.numpy(), v.numpy(), do.numpy(), l, c)
    for a, b in zip(g, g2):
        np.testing.assert_allclose(a, b, atol=1e-11)


def test_row_sampled_entry_points_match_full(orc):
    B, H, T, d = 2, 3, 160, 8
    q, k, v, do = _inputs(B, H, T, d, 9)
    rng = np.random.default_rng(0)
    for kind, mode, l, c in [("fixed", "split", 16, 4), ("strided", "merged", 20, 1)]:
        o, lse = orc.forward(kind, mode, q.numpy(), k.numpy(), v.numpy(), l, c)
        dq, dk, dv = orc.backward(kind, mode, q.numpy(), k.numpy(), v.numpy(), do.numpy(), l, c)
        bh = rng.integers(0, B * H, 40)
        rows = rng.integers(0, T, 40)
        o_r, lse_r = orc.forward_rows(kind, mode, q.numpy(), k.numpy(), v.numpy(), l, c, bh, rows)
        of = o.reshape(B * H, T, d)
        np.testing.assert_allclose(o_r, of[bh, rows], atol=1e-13)
        np.testing.assert_array_equal(lse_r, lse.reshape(B * H, T)[bh, rows])
        dq_r = orc.backward_query_rows(kind, mode, q.numpy(), k.numpy(), v.numpy(), do.numpy(),
                                       l, c, bh, rows)
        np.testing.assert_allclose(dq_r, dq.reshape(B * H, T, d)[bh, rows], atol=1e-12)
        dk_r, dv_r = orc.backward_key_rows(kind, mode, q.numpy(), k.numpy(), v.numpy(),
                                           do.numpy(), l, c, bh, rows)
        np.testing.assert_allclose(dk_r, dk.reshape(B * H, T, d)[bh, rows], atol=1e-12)
        np.testing.assert_allclose(dv_r, dv.reshape(B * H, T, d)[bh, rows], atol=1e-12)


# ---- the oracle's tile derivation ------------------------------------------

@pytest.mark.parametrize("kind,mode,T,l,c", [
    ("fixed", "split", 1024, 64, 8), ("fixed", "merged", 1536, 128, 8),
    ("strided", "split", 1536, 192, 1), ("strided", "merged", 2048, 256, 1),
    ("dense", "merged", 640, 1, 1), ("strided", "merged", 512, 600, 1),
    ("fixed", "merged", 768, 96, 3)])
def test_oracle_tiles_cover_every_pair_once(orc, kind, mode, T, l, c):
    """Per head class, the live counts of all segments add up to the closed-form
    total, and so do those of the plain natural tiling."""
    for hc in range(orc.num_head_classes(kind, mode)):
        if kind == "dense":
            total = T * (T + 1) // 2
        elif kind == "strided":
            total = sum(strided_counts(i, l)[2 if mode == "merged" else hc] for i in range(T))
        else:
            total = sum(fixed_counts(i, l, c)[2 if mode == "merged" else hc] for i in range(T))
        s = 0
        for seg in range(orc.num_segments(kind, mode)):
            _, _, live = orc.layout_tiles(kind, mode, T, l, c, hc, seg)
            assert np.all(live > 0) and np.all(live <= 128 * 128)
            s += int(live.sum())
        assert s == total
        _, _, live = orc.layout_tiles(kind, mode, T, l, c, hc, -1)
        assert int(live.sum()) == total
