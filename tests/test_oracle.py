"""Pins for the fp64 oracle: brute force, closed forms, invariants and library
special cases.  Each one would fail for a plausible slip in the oracle (a
dropped mask, a wrong scale, a transposed operand, a wrong pooling divisor, a
wrong tie rule)."""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O

RNG = np.random.default_rng(1234)


def _rand(*shape, rng=RNG, scale=1.0):
    return rng.standard_normal(shape) * scale


# ---------------------------------------------------------------- budgets


@pytest.mark.parametrize("e,num,den", [(2048, 10, 100), (32768, 10, 100), (65536, 10, 100),
                                       (32, 10, 100), (1, 5, 100), (33, 20, 100), (100, 1, 1),
                                       (131072, 5, 100), (7, 1, 3)])
def test_topk_count_is_exact_ceiling(e, num, den):
    assert O.topk_count(e, num, den) == math.ceil(Fraction(num, den) * e)


def test_topk_count_examples():
    # k = ceil(0.1 N) at the decode context lengths used by the workloads
    assert O.topk_count(2048, 10, 100) == 205
    assert O.topk_count(32768, 10, 100) == 3277
    assert O.topk_count(65536, 10, 100) == 6554


def test_tile_ends_and_offsets():
    assert O.tile_ends(100, 32) == [32, 64, 96, 100]
    ks = O.tile_topk_counts(100, 32, 10, 100)
    assert ks == [4, 7, 10, 10]
    off = O.index_offsets(100, 32, 10, 100)
    assert off.tolist() == [0, 4, 11, 21, 31]


# ---------------------------------------------------------------- Top-k


def _brute_topk(vals, k):
    """Among all k-subsets of maximal total, the lexicographically smallest
    ascending index tuple (lower indices win ties)."""
    best = None
    for sub in itertools.combinations(range(len(vals)), k):
        tot = sum(vals[i] for i in sub)
        key = (-tot, sub)
        if best is None or key < best:
            best = key
    return list(best[1])


@pytest.mark.parametrize("trial", range(40))
def test_select_topk_brute_force_with_ties(trial):
    rng = np.random.default_rng(trial)
    n = int(rng.integers(1, 13))
    k = int(rng.integers(1, n + 1))
    vals = [Fraction(int(x)) for x in rng.integers(0, 4, size=n)]   # many exact ties
    got = O.select_topk(np.array([float(v) for v in vals]), k)
    assert got.tolist() == _brute_topk(vals, k)


@pytest.mark.parametrize("trial", range(20))
def test_select_topk_brute_force_distinct(trial):
    rng = np.random.default_rng(100 + trial)
    n = int(rng.integers(2, 15))
    k = int(rng.integers(1, n + 1))
    vals = rng.random(n)
    got = O.select_topk(vals, k)
    assert got.tolist() == _brute_topk([Fraction(float(v)) for v in vals], k)


def test_selected_set_maximises_pooled_mass():
    q = _rand(1, 8, 1, 32)
    k = _rand(1, 2, 300, 32, scale=1.5)
    idx, pooled = O.anchor_select_decode(q, k, 10, 100)
    for h in range(2):
        sel = set(idx[0, h].tolist())
        inside = min(pooled[0, h, j] for j in sel)
        outside = max(pooled[0, h, j] for j in range(300) if j not in sel)
        assert inside >= outside          # no single swap raises the mass


# ---------------------------------------------------------------- pooling


@pytest.mark.parametrize("n_ctx,tile", [(70, 32), (64, 32), (5, 32), (96, 16)])
def test_pooled_prefill_sums_to_one(n_ctx, tile):
    q = _rand(1, 4, n_ctx, 16)
    k = _rand(1, 2, n_ctx, 16)
    for t in range(-(-n_ctx // tile)):
        for h in range(2):
            p = O.pooled_prefill_tile(q, k, 0, h, t, tile)
            assert p.shape[0] == min(tile * (t + 1), n_ctx)
            assert abs(p.sum() - 1.0) < 1e-12
            assert np.all(p >= 0)


def test_pooled_decode_sums_to_one():
    q = _rand(2, 8, 1, 16)
    k = _rand(2, 4, 50, 16)
    for b in range(2):
        for h in range(4):
            assert abs(O.pooled_decode(q, k, b, h).sum() - 1.0) < 1e-12


def test_q_zero_prefill_closed_form():
    """Q = 0: every visible probability in row i is 1/(i+1), so
    P[j] = (1/rows) * sum over the tile's rows i >= j of 1/(i+1)."""
    n_ctx, tile, d = 80, 32, 8
    q = np.zeros((1, 4, n_ctx, d))
    k = _rand(1, 2, n_ctx, d)
    for t in range(3):
        i0, i1 = t * tile, min(t * tile + tile, n_ctx)
        p = O.pooled_prefill_tile(q, k, 0, 1, t, tile)
        for j in range(i1):
            want = sum(Fraction(1, i + 1) for i in range(max(i0, j), i1)) / (i1 - i0)
            assert abs(p[j] - float(want)) < 1e-15
        # every key before the tile is tied, keys inside get less: ties -> 0..k-1
        kt = O.topk_count(i1, 10, 100)
        idx, _ = O.anchor_select_prefill_tile(q, k, 0, 1, t, tile, 10, 100)
        if kt <= i0:
            assert idx.tolist() == list(range(kt))


def test_q_zero_decode_closed_form():
    """Q = 0: pooled scores are uniform 1/N, the lowest k indices win and the
    output is the plain mean of V_0..V_{k-1} with lse = log k."""
    n_ctx, d = 123, 16
    q = np.zeros((1, 8, 1, d))
    k = _rand(1, 2, n_ctx, d)
    v = _rand(1, 2, n_ctx, d)
    idx, pooled = O.anchor_select_decode(q, k, 10, 100)
    kk = O.topk_count(n_ctx, 10, 100)
    assert np.allclose(pooled, 1.0 / n_ctx, rtol=0, atol=1e-16)
    assert idx[0, 0].tolist() == list(range(kk))
    o, lse = O.sparse_decode(q, k, v, idx)
    for qh in range(8):
        assert np.allclose(o[0, qh], v[0, qh // 4, :kk].mean(0), atol=1e-14)
        assert abs(lse[0, qh] - math.log(kk)) < 1e-13


def test_g1_tile1_is_per_query_topk():
    """G = 1 and tile = 1: the pooled score of tile t is row t's own softmax,
    so the selection is the top-k raw dot products among keys j <= t."""
    n_ctx, d = 40, 8
    q = _rand(1, 1, n_ctx, d)
    k = _rand(1, 1, n_ctx, d)
    for t in range(n_ctx):
        idx, _ = O.anchor_select_prefill_tile(q, k, 0, 0, t, 1, 25, 100)
        raw = [(-float(np.dot(q[0, 0, t], k[0, 0, j])), j) for j in range(t + 1)]
        want = sorted(j for _, j in sorted(raw)[: O.topk_count(t + 1, 25, 100)])
        assert idx.tolist() == want


# ---------------------------------------------------------------- attention


def _sdpa(qr, kr, vr, causal_pos=None):
    qt = torch.tensor(qr)[None, None]
    kt = torch.tensor(kr)[None, None]
    vt = torch.tensor(vr)[None, None]
    mask = None
    if causal_pos is not None:
        mask = torch.tensor(np.arange(kr.shape[0])[None, :] <= np.asarray(causal_pos)[:, None])
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)[0, 0].numpy()


def test_dense_matches_torch_sdpa():
    qr, kr, vr = _rand(5, 32), _rand(40, 32), _rand(40, 32)
    o, _ = O.dense_attention(qr, kr, vr)
    assert np.allclose(o, _sdpa(qr, kr, vr), atol=1e-12)
    pos = np.array([0, 3, 17, 39, 25])
    o, _ = O.dense_attention(qr, kr, vr, pos)
    assert np.allclose(o, _sdpa(qr, kr, vr, pos), atol=1e-12)


def test_lse_matches_logsumexp():
    qr, kr, vr = _rand(3, 16), _rand(20, 16), _rand(20, 16)
    _, lse = O.dense_attention(qr, kr, vr)
    s = torch.tensor(qr) @ torch.tensor(kr).T / 4.0
    assert np.allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12)


def test_frac_one_decode_equals_dense():
    q = _rand(2, 8, 1, 16)
    k, v = _rand(2, 2, 37, 16), _rand(2, 2, 37, 16)
    idx, _ = O.anchor_select_decode(q, k, 1, 1)
    assert idx.shape[-1] == 37
    o, _ = O.sparse_decode(q, k, v, idx)
    for b in range(2):
        for qh in range(8):
            want = _sdpa(q[b, qh], k[b, qh // 4], v[b, qh // 4])
            assert np.allclose(o[b, qh], want[0], atol=1e-12)


def test_frac_one_prefill_equals_causal_dense():
    n_ctx, tile = 45, 16
    q = _rand(1, 4, n_ctx, 8)
    k, v = _rand(1, 2, n_ctx, 8), _rand(1, 2, n_ctx, 8)
    for t in range(3):
        for h in range(2):
            sel, _ = O.anchor_select_prefill_tile(q, k, 0, h, t, tile, 1, 1)
            o, _ = O.sparse_prefill_tile(q, k, v, sel, 0, h, t, tile)
            i0, i1 = t * tile, min(t * tile + tile, n_ctx)
            for g in range(2):
                want = _sdpa(q[0, 2 * h + g], k[0, h], v[0, h], np.arange(n_ctx))[i0:i1]
                assert np.allclose(o[g], want, atol=1e-12)


def test_single_key_outputs_v0():
    q = _rand(1, 4, 1, 8)
    k, v = _rand(1, 1, 1, 8), _rand(1, 1, 1, 8)
    idx, _ = O.anchor_select_decode(q, k, 10, 100)
    o, lse = O.sparse_decode(q, k, v, idx)
    assert np.allclose(o[0], v[0, 0, 0][None, :], atol=1e-15)
    qp = _rand(1, 4, 1, 8)
    sel, _ = O.anchor_select_prefill_tile(qp, k, 0, 0, 0, 32, 10, 100)
    o, _ = O.sparse_prefill_tile(qp, k, v, sel, 0, 0, 0, 32)
    assert np.allclose(o[:, 0], v[0, 0, 0][None, :], atol=1e-15)


def test_two_keys_logistic():
    """Two keys: the weight of key 0 is the logistic function of the score gap."""
    d = 4
    q = np.array([[[[1.0, 2.0, 0.0, -1.0]]]])
    k = np.array([[[[0.5, 0.5, 1.0, 0.0], [-1.0, 1.0, 0.0, 2.0]]]])
    v = np.array([[[[1.0, 0.0, 0.0, 0.0], [0.0, 1.0, 0.0, 0.0]]]])
    gap = ((1.5) - (-1.0)) / math.sqrt(d)     # (q.k0 - q.k1) / sqrt(d), worked by hand
    w0 = 1.0 / (1.0 + math.exp(-gap))
    o, _ = O.sparse_decode(q, k, v, np.array([[[0, 1]]]))
    assert np.allclose(o[0, 0], [w0, 1 - w0, 0, 0], atol=1e-15)


def test_prefill_row_without_visible_key():
    """A row whose selected keys all lie in its future outputs 0, lse -inf."""
    q = _rand(1, 1, 4, 4)
    k, v = _rand(1, 1, 4, 4), _rand(1, 1, 4, 4)
    o, lse = O.sparse_prefill_tile(q, k, v, np.array([2, 3]), 0, 0, 0, 4)
    assert np.all(o[0, :2] == 0) and np.all(np.isneginf(lse[0, :2]))
    assert np.all(np.isfinite(lse[0, 2:]))


# ---------------------------------------------------------------- head-aware reuse


def test_head_permutation_equivariance():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 8, 1, 16))
    k = rng.standard_normal((1, 4, 60, 16))
    v = rng.standard_normal((1, 4, 60, 16))
    perm = np.array([2, 0, 3, 1])
    qperm = q.reshape(1, 4, 2, 1, 16)[:, perm].reshape(1, 8, 1, 16)
    idx, _ = O.anchor_select_decode(q, k, 20, 100)
    idx_p, _ = O.anchor_select_decode(qperm, k[:, perm], 20, 100)
    assert np.array_equal(idx_p, idx[:, perm])
    o, _ = O.sparse_decode(q, k, v, idx)
    o_p, _ = O.sparse_decode(qperm, k[:, perm], v[:, perm], idx_p)
    assert np.allclose(o_p.reshape(1, 4, 2, 16), o.reshape(1, 4, 2, 16)[:, perm], atol=1e-13)


def test_reuse_of_own_anchor_reproduces_anchor():
    q = _rand(1, 8, 1, 16)
    k, v = _rand(1, 2, 90, 16), _rand(1, 2, 90, 16)
    idx, _ = O.anchor_select_decode(q, k, 10, 100)
    o_anchor, _ = O.sparse_decode(q, k, v, idx, None)
    o_reuse, _ = O.sparse_decode(q, k, v, idx, [0, 1])
    assert np.array_equal(o_anchor, o_reuse)


def test_head_map_reads_mapped_anchor_set():
    """head_map [1, 1]: both kv heads use anchor head 1's set, which for head 1
    is its own set and for head 0 equals attending over those positions."""
    q = _rand(1, 4, 1, 8)
    k, v = _rand(1, 2, 50, 8), _rand(1, 2, 50, 8)
    idx = np.array([[[1, 5, 9], [0, 7, 30]]])
    o, _ = O.sparse_decode(q, k, v, idx, [1, 1])
    want0, _ = O.dense_attention(q[0, 0:2, 0], k[0, 0, [0, 7, 30]], v[0, 0, [0, 7, 30]])
    assert np.allclose(o[0, 0:2], want0, atol=1e-14)


# ---------------------------------------------------------------- acceptance rule


def test_check_index_set_rules():
    p = np.array([0.5, 0.2, 0.2 * (1 - 1e-7), 0.05, 0.05])
    assert O.check_index_set(p, 2, [0, 1]) == "exact"
    assert O.check_index_set(p, 2, [0, 2]) == "near_tie"
    assert O.check_index_set(p, 2, [0, 3]) == "fail"
    assert O.check_index_set(p, 2, [1, 2]) == "fail"   # drops the clear winner
    q = np.array([0.5, 0.2, 0.1, 0.05])
    assert O.check_index_set(q, 2, [0, 2]) == "fail"   # gap far above the tie band
    assert O.check_index_set(q, 2, [1, 0]) == "fail"   # not ascending
