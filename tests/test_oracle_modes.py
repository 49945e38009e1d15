"""Pins for the oracle's head-selection variants (per query head, the
oracle_topk strategy; all heads pooled, the head-unaware strategy): exact
closed forms for Q = 0, linearity of the post-softmax mean across the three
poolings, per-head selection by raw score (softmax is monotone), the
special cases where two modes coincide, and frac = 1 against torch's SDPA.
Also the proposal-refine selection: the whole context as the pool gives the
anchor selection, a pool of kappa keys is returned as is, Q = 0 takes the
lowest pool entries, and brute force over a small pool (softmax by torch)."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O

RNG = np.random.default_rng(77)


def _qkv(B, Hq, Hkv, L, N, d, scale=1.0):
    q = RNG.standard_normal((B, Hq, L, d)) * scale
    k = RNG.standard_normal((B, Hkv, N, d))
    v = RNG.standard_normal((B, Hkv, N, d))
    return q, k, v


def test_selection_heads_partition():
    assert O.selection_heads(8, 2, "gqa") == [[0, 1, 2, 3], [4, 5, 6, 7]]
    assert O.selection_heads(8, 2, "head") == [[i] for i in range(8)]
    assert O.selection_heads(8, 2, "all") == [list(range(8))]
    with pytest.raises(ValueError):
        O.selection_heads(8, 2, "rows")


@pytest.mark.parametrize("mode", O.MODES)
def test_q_zero_decode_is_uniform_and_takes_lowest_indices(mode):
    B, Hq, Hkv, N, d = 2, 6, 2, 37, 16
    q = np.zeros((B, Hq, 1, d))
    k = RNG.standard_normal((B, Hkv, N, d))
    idx, pooled = O.anchor_select_decode_mode(q, k, 10, 100, mode)
    assert np.allclose(pooled, 1.0 / N, rtol=0, atol=1e-15)
    kk = O.topk_count(N, 10, 100)
    assert (idx == np.arange(kk)).all()


@pytest.mark.parametrize("mode", O.MODES)
def test_q_zero_prefill_exact_rational(mode):
    """Q = 0: row i gives 1/(i+1) to each key j <= i, in every head, so any
    pooling over heads gives P[j] = (1/rows) sum_{i in tile, i >= j} 1/(i+1)."""
    B, Hq, Hkv, N, d, tile = 1, 4, 2, 70, 8, 32
    q = np.zeros((B, Hq, N, d))
    k = RNG.standard_normal((B, Hkv, N, d))
    n_prob = len(O.selection_heads(Hq, Hkv, mode))
    for t in range(3):
        i0, i1 = 32 * t, min(32 * t + 32, N)
        want = [float(sum((Fraction(1, i + 1) for i in range(max(i0, j), i1)), Fraction(0)) / (i1 - i0))
                for j in range(i1)]
        for p in range(n_prob):
            _, pooled = O.anchor_select_prefill_tile_mode(q, k, 0, p, t, tile, 10, 100, mode)
            assert np.allclose(pooled, want, rtol=0, atol=1e-15)


def test_pooling_is_linear_across_modes_decode():
    """Per-head pooled values averaged over a GQA group give that group's
    pooled values; GQA values averaged over kv heads give the all-heads
    values (the post-softmax mean is linear)."""
    B, Hq, Hkv, N, d = 2, 8, 2, 50, 32
    q, k, _ = _qkv(B, Hq, Hkv, 1, N, d, scale=0.7)
    G = Hq // Hkv
    _, ph = O.anchor_select_decode_mode(q, k, 10, 100, "head")
    _, pg = O.anchor_select_decode_mode(q, k, 10, 100, "gqa")
    _, pa = O.anchor_select_decode_mode(q, k, 10, 100, "all")
    for b in range(B):
        for h in range(Hkv):
            assert np.allclose(ph[b, h * G:(h + 1) * G].mean(axis=0), pg[b, h], rtol=1e-13, atol=0)
            # and the gqa mode agrees with the default-path function
            assert np.allclose(pg[b, h], O.pooled_decode(q, k, b, h), rtol=1e-13, atol=0)
        assert np.allclose(pg[b].mean(axis=0), pa[b, 0], rtol=1e-13, atol=0)


def test_pooling_is_linear_across_modes_prefill():
    B, Hq, Hkv, N, d = 1, 4, 2, 80, 16
    q, k, _ = _qkv(B, Hq, Hkv, N, N, d, scale=0.5)
    for t in range(3):
        per_head = [O.anchor_select_prefill_tile_mode(q, k, 0, p, t, 32, 10, 100, "head")[1] for p in range(Hq)]
        gqa = [O.anchor_select_prefill_tile_mode(q, k, 0, p, t, 32, 10, 100, "gqa")[1] for p in range(Hkv)]
        allh = O.anchor_select_prefill_tile_mode(q, k, 0, 0, t, 32, 10, 100, "all")[1]
        for h in range(Hkv):
            assert np.allclose(np.mean(per_head[2 * h:2 * h + 2], axis=0), gqa[h], rtol=1e-13, atol=0)
            assert np.allclose(gqa[h], O.pooled_prefill_tile(q, k, 0, h, t, 32), rtol=1e-13, atol=0)
        assert np.allclose(np.mean(gqa, axis=0), allh, rtol=1e-13, atol=0)


def test_head_mode_selects_largest_raw_scores():
    """One decode query per head: softmax is monotone, so the per-head set
    is the k largest raw scores q . k_j (lower index on ties)."""
    B, Hq, Hkv, N, d = 2, 6, 3, 64, 8
    q, k, _ = _qkv(B, Hq, Hkv, 1, N, d)
    k[:, :, 10] = k[:, :, 11]          # an exact tie between two keys
    idx, _ = O.anchor_select_decode_mode(q, k, 25, 100, "head")
    kk = O.topk_count(N, 25, 100)
    G = Hq // Hkv
    for b in range(B):
        for qh in range(Hq):
            raw = k[b, qh // G] @ q[b, qh, 0]
            order = sorted(range(N), key=lambda j: (-raw[j], j))[:kk]
            assert idx[b, qh].tolist() == sorted(order)


def test_all_mode_with_one_kv_head_is_gqa():
    B, Hq, Hkv, N, d = 2, 4, 1, 40, 8
    q, k, _ = _qkv(B, Hq, Hkv, 1, N, d)
    ia, pa = O.anchor_select_decode_mode(q, k, 10, 100, "all")
    ig, pg = O.anchor_select_decode_mode(q, k, 10, 100, "gqa")
    assert (ia == ig).all() and np.array_equal(pa, pg)


def test_head_mode_with_group_of_one_is_gqa():
    B, Hq, Hkv, N, d = 1, 3, 3, 45, 8
    q, k, _ = _qkv(B, Hq, Hkv, 1, N, d)
    ih, ph = O.anchor_select_decode_mode(q, k, 20, 100, "head")
    ig, pg = O.anchor_select_decode_mode(q, k, 20, 100, "gqa")
    assert (ih == ig).all() and np.allclose(ph, pg, rtol=1e-15, atol=0)


def test_sparse_decode_modes_reduce_to_the_default_path():
    B, Hq, Hkv, N, d = 2, 8, 2, 60, 16
    q, k, v = _qkv(B, Hq, Hkv, 1, N, d)
    G = Hq // Hkv
    idx_g, _ = O.anchor_select_decode_mode(q, k, 20, 100, "gqa")
    hm = [1, 0]
    want, wl = O.sparse_decode(q, k, v, idx_g, hm)
    got, gl = O.sparse_decode_mode(q, k, v, idx_g, "gqa", hm)
    assert np.allclose(got, want, rtol=1e-14, atol=1e-14) and np.allclose(gl, wl, rtol=1e-14)
    # head mode whose per-head lists are the group's list and whose head map
    # sends query head qh to the head that holds group hm[qh // G]'s list
    idx_h = np.repeat(idx_g, G, axis=1)
    hm_h = [hm[qh // G] * G for qh in range(Hq)]
    got, _ = O.sparse_decode_mode(q, k, v, idx_h, "head", hm_h)
    assert np.allclose(got, want, rtol=1e-14, atol=1e-14)
    # all mode: one list per batch row, read by every head
    one = idx_g[:, :1]
    want1, _ = O.sparse_decode(q, k, v, np.repeat(one, Hkv, axis=1))
    got1, _ = O.sparse_decode_mode(q, k, v, one, "all", None)
    assert np.allclose(got1, want1, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("mode", O.MODES)
def test_frac_one_modes_equal_sdpa(mode):
    """frac = 1 selects every key in every mode: decode equals dense
    attention and prefill causal dense attention (torch fp64 SDPA)."""
    B, Hq, Hkv, N, d = 1, 4, 2, 40, 8
    G = Hq // Hkv
    q, k, v = _qkv(B, Hq, Hkv, 1, N, d)
    idx, _ = O.anchor_select_decode_mode(q, k, 1, 1, mode)
    o, _ = O.sparse_decode_mode(q, k, v, idx, mode)
    kt = torch.from_numpy(np.repeat(k, G, axis=1))
    vt = torch.from_numpy(np.repeat(v, G, axis=1))
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q), kt, vt)
    assert np.allclose(o, ref[:, :, 0].numpy(), rtol=1e-12, atol=1e-12)
    qp, kp, vp = _qkv(B, Hq, Hkv, N, N, d)
    n_prob = len(O.selection_heads(Hq, Hkv, mode))
    refp = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(qp), torch.from_numpy(np.repeat(kp, G, axis=1)),
        torch.from_numpy(np.repeat(vp, G, axis=1)), is_causal=True).numpy()
    for t in range(2):
        lists = [O.anchor_select_prefill_tile_mode(qp, kp, 0, p, t, 32, 1, 1, mode)[0] for p in range(n_prob)]
        op, _ = O.sparse_prefill_tile_mode(qp, kp, vp, lists, 0, t, 32, mode)
        assert np.allclose(op, refp[0, :, 32 * t:min(32 * t + 32, N)], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- proposal-refine reuse


def test_refine_over_the_whole_context_is_the_anchor_selection():
    B, Hq, Hkv, N, d = 2, 8, 2, 90, 16
    q, k, _ = _qkv(B, Hq, Hkv, 1, N, d)
    kk = O.topk_count(N, 10, 100)
    pool = np.tile(np.arange(N), (B, Hkv, 1))
    idx, pooled = O.refine_select_decode(q, k, pool, kk)
    want, wp = O.anchor_select_decode(q, k, 10, 100)
    assert (idx == want).all() and np.allclose(pooled, wp, rtol=1e-14, atol=0)


def test_refine_with_a_pool_of_kappa_returns_the_pool():
    B, Hq, Hkv, N, d = 1, 4, 2, 50, 8
    q, k, _ = _qkv(B, Hq, Hkv, 1, N, d)
    pool = np.stack([[np.sort(RNG.choice(N, 7, replace=False)) for _ in range(Hkv)] for _ in range(B)])
    idx, _ = O.refine_select_decode(q, k, pool, 7)
    assert (idx == pool).all()


def test_refine_q_zero_takes_the_lowest_pool_entries():
    """Q = 0: uniform over the pool, so ties everywhere and the kappa lowest
    key indices of the pool win."""
    B, Hq, Hkv, N, d = 1, 4, 2, 64, 8
    q = np.zeros((B, Hq, 1, d))
    k = RNG.standard_normal((B, Hkv, N, d))
    pool = np.stack([[np.sort(RNG.choice(N, 20, replace=False)) for _ in range(Hkv)] for _ in range(B)])
    idx, pooled = O.refine_select_decode(q, k, pool, 5, head_map=[1, 0])
    assert np.allclose(pooled, 1.0 / 20, rtol=0, atol=1e-15)
    assert (idx[0, 0] == pool[0, 1, :5]).all() and (idx[0, 1] == pool[0, 0, :5]).all()


def test_refine_brute_force_pool_mass():
    """The refined set maximises the pooled mass (softmax over the pool) over
    all kappa-subsets of a small pool; ties go to lower key indices."""
    import itertools
    B, Hq, Hkv, N, d = 1, 4, 1, 40, 4
    for trial in range(5):
        q, k, _ = _qkv(B, Hq, Hkv, 1, N, d)
        cand = np.sort(RNG.choice(N, 10, replace=False))
        # pooled over the pool, computed independently with torch
        qt = torch.from_numpy(q[0, :, 0])
        kt = torch.from_numpy(k[0, 0, cand])
        p = torch.softmax(qt @ kt.T / np.sqrt(d), dim=-1).mean(0).numpy()
        best = max(itertools.combinations(range(10), 3), key=lambda sub: (round(sum(p[list(sub)]), 15), [-i for i in sub]))
        idx, _ = O.refine_select_decode(q, k, cand[None, None, :], 3)
        assert idx[0, 0].tolist() == cand[list(best)].tolist()


# ---------------------------------------------------------------- anchor-layer selection


def _brute_plan(sim, m):
    """Exhaustive: every anchor set containing layer 0; each layer reuses its
    nearest preceding anchor; best total, lexicographically smallest set on
    ties."""
    import itertools
    n = sim.shape[0]
    best = None
    for rest in itertools.combinations(range(1, n), m - 1):
        anchors = (0,) + rest
        tot = 0.0
        for l in range(n):
            a = max(x for x in anchors if x <= l)
            tot += sim[a, l]
        if best is None or tot > best[1] + 1e-12 or (abs(tot - best[1]) <= 1e-12 and anchors < best[0]):
            best = (anchors, tot)
    return list(best[0]), best[1]


@pytest.mark.parametrize("n,m", [(6, 1), (6, 2), (7, 3), (8, 4), (9, 9), (10, 3)])
def test_plan_anchors_brute_force(n, m):
    for trial in range(4):
        sim = np.triu(RNG.random((n, n)))
        np.fill_diagonal(sim, 1.0)
        got = O.plan_anchors(sim, m)
        want = _brute_plan(sim, m)
        assert got[0] == want[0] and abs(got[1] - want[1]) < 1e-12


def test_plan_anchors_closed_forms():
    # identical layers: any plan scores n; the smallest anchor set wins
    sim = np.ones((5, 5))
    assert O.plan_anchors(sim, 3) == ([0, 1, 2], 5.0)
    # two blocks of mutually similar layers: the second block's first layer
    sim = np.zeros((6, 6))
    sim[:3, :3] = 1.0
    sim[3:, 3:] = 1.0
    assert O.plan_anchors(sim, 2) == ([0, 3], 6.0)
    # every layer its own anchor
    assert O.plan_anchors(np.eye(4), 4) == ([0, 1, 2, 3], 4.0)
    with pytest.raises(ValueError):
        O.plan_anchors(np.eye(3), 0)


def test_index_overlap_counts():
    assert O.index_overlap([1, 3, 5, 7], [0, 3, 4, 7, 9]) == 2
    assert O.index_overlap([], [1, 2]) == 0
    assert O.index_overlap(np.arange(10), np.arange(5, 20)) == 5
