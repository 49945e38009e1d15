"""Kascade oracle: a plain, slow fp64 CPU statement of head-aware, cross-layer
reused Top-k sparse attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code with the CUDA library.

Sources (page "A Practical Sparse Attention Method for Long-Context LLM
Inference", the Kascade README):

* Abstract: post-softmax attention is sparse; exact Top-k indices are computed
  in a few *anchor* layers and reused by the *reuse* layers in between;
  selection and reuse are head-aware; operations are tile-level in prefill and
  decode.
* "Running Evaluations and Performance Benchmarks": the selection strategy is
  ``post_softmax_pooled_prefill_topk`` and the efficient kernels use
  ``tile_size 32``; the figure caption under the Abstract and the ``--topk 10``
  / ``k=10`` arguments ("Kernel Benchmarks", "Python API") give the budget as a
  percentage of the context.

Readings of what the page leaves open:

* scores are q.k / sqrt(d) with no bias (standard scaled dot product);
* query head qh belongs to kv head qh // G (contiguous GQA groups);
* "pooled" = the mean of post-softmax probabilities over the G query heads of
  a kv head and, in prefill, over the rows of one query tile; masked
  (future) entries count as 0 and the mean is over all G*rows entries;
* k = ceil(frac * e) computed in integers, frac = num/den; e = the number of
  candidate keys (decode: N; prefill tile t: min(tile*(t+1), N));
* the k largest pooled values win; equal values go to the lower key index;
  index lists are reported in ascending order;
* decode: the single query sees all N cached keys;
* prefill: the candidates of tile t are keys [0, e_t); row i attends only to
  selected keys j <= i; a row that sees no selected key outputs 0 with
  log-sum-exp -inf;
* a reuse kv head h reads the index set of anchor head head_map[h].

Everything is computed in float64 from the exact values of the (bf16) inputs.
Array layout: q [B, Hq, L, d], k/v [B, Hkv, N, d] (L = 1 in decode).
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64

__all__ = [
    "topk_count", "tile_ends", "tile_topk_counts", "index_offsets",
    "scores", "masked_softmax", "pooled_decode", "pooled_prefill_tile",
    "select_topk", "anchor_select_decode", "anchor_select_prefill_tile",
    "sparse_attend", "sparse_decode", "sparse_prefill_tile", "dense_attention",
    "check_index_set",
    "MODES", "selection_heads", "pooled_decode_heads", "pooled_prefill_tile_heads",
    "anchor_select_decode_mode", "anchor_select_prefill_tile_mode", "sparse_decode_mode",
    "sparse_prefill_tile_mode", "refine_select_decode", "index_overlap", "plan_anchors",
]


# ---------------------------------------------------------------------------
# budgets and tiles


def topk_count(e: int, frac_num: int, frac_den: int) -> int:
    """k = ceil(frac * e) with frac = frac_num / frac_den, in exact integers.

    The README gives the budget as a percentage ("Top-k set to 10%", Abstract
    figure caption; ``--topk 10``, Kernel Benchmarks)."""
    if e <= 0:
        return 0
    return -((-frac_num * e) // frac_den)


def tile_ends(n_ctx: int, tile: int) -> list[int]:
    """e_t = min(tile*(t+1), N) for t = 0..ceil(N/tile)-1: the keys that the
    last row of query tile t can see (tile-level prefill, README Abstract)."""
    n_tiles = -(-n_ctx // tile)
    return [min(tile * (t + 1), n_ctx) for t in range(n_tiles)]


def tile_topk_counts(n_ctx: int, tile: int, frac_num: int, frac_den: int) -> list[int]:
    """k_t for every prefill tile."""
    return [topk_count(e, frac_num, frac_den) for e in tile_ends(n_ctx, tile)]


def index_offsets(n_ctx: int, tile: int, frac_num: int, frac_den: int) -> np.ndarray:
    """Start of each tile's index list in a ragged [sum_t k_t] row (plus the
    total at the end)."""
    ks = tile_topk_counts(n_ctx, tile, frac_num, frac_den)
    out = np.zeros(len(ks) + 1, dtype=np.int64)
    out[1:] = np.cumsum(ks)
    return out


# ---------------------------------------------------------------------------
# scores, softmax, pooling


def scores(q_rows: np.ndarray, k_rows: np.ndarray) -> np.ndarray:
    """s[r, j] = q_r . k_j / sqrt(d) in float64."""
    q64 = np.asarray(q_rows, dtype=F64)
    k64 = np.asarray(k_rows, dtype=F64)
    return (q64 @ k64.T) / math.sqrt(q64.shape[-1])


def masked_softmax(s: np.ndarray, visible: np.ndarray) -> np.ndarray:
    """Row softmax over the visible entries; invisible entries are 0.  A row
    with nothing visible is all zeros."""
    s = np.where(visible, s, -np.inf)
    m = np.max(s, axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    p = np.where(visible, np.exp(s - m), 0.0)
    den = p.sum(axis=-1, keepdims=True)
    return np.divide(p, den, out=np.zeros_like(p), where=den > 0)


def pooled_decode(q: np.ndarray, k: np.ndarray, b: int, h: int) -> np.ndarray:
    """Pooled post-softmax scores of kv head h for one decode query.

    P[j] = (1/G) sum_g softmax_j(q_{hG+g} . k_j / sqrt(d)), j < N."""
    hq, hkv = q.shape[1], k.shape[1]
    g_size = hq // hkv
    q_rows = q[b, h * g_size:(h + 1) * g_size, 0, :]
    s = scores(q_rows, k[b, h])
    p = masked_softmax(s, np.ones_like(s, dtype=bool))
    return p.mean(axis=0)


def pooled_prefill_tile(q: np.ndarray, k: np.ndarray, b: int, h: int, t: int,
                        tile: int) -> np.ndarray:
    """Pooled post-softmax scores of kv head h over query tile t.

    Rows are the G heads x the tile's query positions i; candidates are keys
    j < e_t; row i sees j <= i.  P[j] = sum over rows of p[r, j] divided by
    G * rows_t (rows_t = the tile's real rows)."""
    hq, hkv, n_ctx = q.shape[1], k.shape[1], k.shape[2]
    g_size = hq // hkv
    i0 = t * tile
    i1 = min(i0 + tile, n_ctx)
    e_t = i1
    pos = np.arange(i0, i1)
    total = np.zeros(e_t, dtype=F64)
    for g in range(g_size):
        s = scores(q[b, h * g_size + g, i0:i1, :], k[b, h, :e_t, :])
        visible = np.arange(e_t)[None, :] <= pos[:, None]
        total += masked_softmax(s, visible).sum(axis=0)
    return total / (g_size * (i1 - i0))


# ---------------------------------------------------------------------------
# Top-k


def select_topk(pooled: np.ndarray, k: int) -> np.ndarray:
    """The k largest pooled values, equal values going to the lower index,
    returned as ascending indices."""
    n = pooled.shape[0]
    order = np.lexsort((np.arange(n), -np.asarray(pooled, dtype=F64)))
    return np.sort(order[:k]).astype(np.int64)


def anchor_select_decode(q: np.ndarray, k: np.ndarray, frac_num: int, frac_den: int):
    """Anchor decode layer: idx [B, Hkv, kk] (ascending) and pooled [B, Hkv, N]."""
    bsz, hkv, n_ctx = k.shape[0], k.shape[1], k.shape[2]
    kk = topk_count(n_ctx, frac_num, frac_den)
    idx = np.zeros((bsz, hkv, kk), dtype=np.int64)
    pooled = np.zeros((bsz, hkv, n_ctx), dtype=F64)
    for b in range(bsz):
        for h in range(hkv):
            pooled[b, h] = pooled_decode(q, k, b, h)
            idx[b, h] = select_topk(pooled[b, h], kk)
    return idx, pooled


def anchor_select_prefill_tile(q, k, b, h, t, tile, frac_num, frac_den):
    """Anchor prefill, one (b, h, t) problem: (ascending idx of k_t keys, pooled)."""
    pooled = pooled_prefill_tile(q, k, b, h, t, tile)
    return select_topk(pooled, topk_count(pooled.shape[0], frac_num, frac_den)), pooled


# ---------------------------------------------------------------------------
# sparse attention over a selected set


def sparse_attend(q_rows: np.ndarray, k_rows: np.ndarray, v_rows: np.ndarray,
                  visible: np.ndarray):
    """o_r = sum_j softmax_j(q_r . k_j / sqrt(d)) v_j over the visible j, with
    log-sum-exp lse_r of the scaled scores.  Rows with nothing visible give
    o = 0 and lse = -inf."""
    s = scores(q_rows, k_rows)
    p = masked_softmax(s, visible)
    o = p @ np.asarray(v_rows, dtype=F64)
    s_vis = np.where(visible, s, -np.inf)
    m = np.max(s_vis, axis=-1)
    has = np.isfinite(m)
    m0 = np.where(has, m, 0.0)
    with np.errstate(divide="ignore"):
        lse = np.where(has, m0 + np.log(np.where(visible, np.exp(s_vis - m0[:, None]), 0.0).sum(-1)),
                       -np.inf)
    return o, lse


def sparse_decode(q, k, v, idx, head_map=None):
    """Reuse (or anchor) decode layer.  kv head h attends over the set
    idx[b, head_map[h]]; head_map None means identity.

    Returns o [B, Hq, d] and lse [B, Hq] (natural log of the softmax
    denominator of the scaled scores)."""
    bsz, hq, _, d = q.shape
    hkv = k.shape[1]
    g_size = hq // hkv
    hm = np.arange(hkv) if head_map is None else np.asarray(head_map)
    o = np.zeros((bsz, hq, d), dtype=F64)
    lse = np.zeros((bsz, hq), dtype=F64)
    for b in range(bsz):
        for h in range(hkv):
            sel = np.asarray(idx[b, hm[h]], dtype=np.int64)
            rows = q[b, h * g_size:(h + 1) * g_size, 0, :]
            vis = np.ones((g_size, sel.shape[0]), dtype=bool)
            ob, lb = sparse_attend(rows, k[b, h, sel], v[b, h, sel], vis)
            o[b, h * g_size:(h + 1) * g_size] = ob
            lse[b, h * g_size:(h + 1) * g_size] = lb
    return o, lse


def sparse_prefill_tile(q, k, v, sel, b, h, t, tile):
    """Reuse (or anchor) prefill, one (b, h, t) problem over the selected set
    ``sel`` (the anchor head's list for tile t).  Row i of the tile sees the
    selected keys j <= i.  Returns o [G, rows_t, d] and lse [G, rows_t]."""
    hq, hkv, n_ctx = q.shape[1], k.shape[1], k.shape[2]
    g_size = hq // hkv
    i0 = t * tile
    i1 = min(i0 + tile, n_ctx)
    sel = np.asarray(sel, dtype=np.int64)
    pos = np.arange(i0, i1)
    vis = sel[None, :] <= pos[:, None]
    o = np.zeros((g_size, i1 - i0, q.shape[-1]), dtype=F64)
    lse = np.zeros((g_size, i1 - i0), dtype=F64)
    for g in range(g_size):
        o[g], lse[g] = sparse_attend(q[b, h * g_size + g, i0:i1, :], k[b, h, sel], v[b, h, sel], vis)
    return o, lse


def dense_attention(q_rows, k_rows, v_rows, row_pos=None):
    """Dense attention of q_rows over all keys (row_pos None) or causally
    (key j visible to the row at position row_pos[r] iff j <= row_pos[r])."""
    n = k_rows.shape[0]
    if row_pos is None:
        vis = np.ones((q_rows.shape[0], n), dtype=bool)
    else:
        vis = np.arange(n)[None, :] <= np.asarray(row_pos)[:, None]
    return sparse_attend(q_rows, k_rows, v_rows, vis)


# ---------------------------------------------------------------------------
# acceptance rule for a selected set


def check_index_set(pooled: np.ndarray, k: int, got, rel: float = 1e-6) -> str:
    """Judge an index set against the oracle's pooled values.

    Let tau_k, tau_k1 be the k-th and (k+1)-th largest pooled values.  If
    tau_k - tau_k1 > rel * tau_k the set must equal the oracle's exactly
    ("exact").  Otherwise (a near tie) it passes ("near_tie") when it holds
    every j with P_j > tau_k (1 + rel) and all of its other members lie
    within rel * tau_k of tau_k.  Anything else is "fail".  The set must also
    be strictly ascending with k members in range."""
    pooled = np.asarray(pooled, dtype=F64)
    got = np.asarray(got, dtype=np.int64)
    n = pooled.shape[0]
    if got.shape[0] != k or (k > 0 and (got.min() < 0 or got.max() >= n)):
        return "fail"
    if k > 1 and not np.all(np.diff(got) > 0):
        return "fail"
    want = select_topk(pooled, k)
    if np.array_equal(want, got):
        return "exact"
    srt = np.sort(pooled)[::-1]
    tau_k = srt[k - 1]
    tau_k1 = srt[k] if k < n else -np.inf
    if tau_k - tau_k1 > rel * tau_k:
        return "fail"
    must = np.nonzero(pooled > tau_k * (1.0 + rel))[0]
    if not np.all(np.isin(must, got)):
        return "fail"
    others = np.setdiff1d(got, must)
    if np.all(np.abs(pooled[others] - tau_k) <= rel * tau_k):
        return "near_tie"
    return "fail"


# ---------------------------------------------------------------------------
# head-selection variants
#
# The README's Reproducibility section runs two more selection strategies
# beside the default post_softmax_pooled_prefill_topk: oracle_topk (Figure 1,
# sparsity "per Layer per Head") and post_softmax_all_heads_pooled_oracle_topk
# (Figure 3).  The Abstract calls head-aware selection critical, which is the
# contrast these variants show.  Readings (the page names the strategies and
# nothing more):
#
# * "gqa"  (default): one problem per kv head h pools the post-softmax
#   probabilities of its G query heads, as everything above;
# * "head" (oracle_topk): one problem per query head qh, no pooling across
#   heads; in prefill the tile-level constraint still holds, so the problem
#   pools the rows of query tile t of that one head;
# * "all"  (all heads pooled): one problem per batch row (and tile) pools
#   every query head of every kv head, each scored against its own kv head's
#   keys; all heads then share the one index set ("head-unaware").
# A reuse layer in "head" mode maps query heads to anchor query heads
# (head_map over [0, Hq)); in "all" mode every head reads the batch's single
# list.

MODES = ("gqa", "head", "all")


def selection_heads(hq: int, hkv: int, mode: str) -> list[list[int]]:
    """The query heads each selection problem of one batch row pools, in
    problem order (gqa: Hkv problems, head: Hq, all: 1)."""
    g_size = hq // hkv
    if mode == "gqa":
        return [list(range(h * g_size, (h + 1) * g_size)) for h in range(hkv)]
    if mode == "head":
        return [[qh] for qh in range(hq)]
    if mode == "all":
        return [list(range(hq))]
    raise ValueError(mode)


def pooled_decode_heads(q: np.ndarray, k: np.ndarray, b: int, heads) -> np.ndarray:
    """P[j] = mean over the listed query heads qh of
    softmax_j(q_qh . k_{qh // G, j} / sqrt(d)), j < N (decode)."""
    hq, hkv, n_ctx = q.shape[1], k.shape[1], k.shape[2]
    g_size = hq // hkv
    total = np.zeros(n_ctx, dtype=F64)
    for qh in heads:
        s = scores(q[b, qh, 0:1, :], k[b, qh // g_size])
        total += masked_softmax(s, np.ones_like(s, dtype=bool))[0]
    return total / len(heads)


def pooled_prefill_tile_heads(q: np.ndarray, k: np.ndarray, b: int, heads, t: int,
                              tile: int) -> np.ndarray:
    """Pooled post-softmax scores of query tile t over the listed query
    heads: candidates j < e_t, row i sees j <= i, each head scored against
    its own kv head's keys, sum over heads and rows divided by
    len(heads) * rows_t."""
    hq, hkv, n_ctx = q.shape[1], k.shape[1], k.shape[2]
    g_size = hq // hkv
    i0 = t * tile
    i1 = min(i0 + tile, n_ctx)
    e_t = i1
    pos = np.arange(i0, i1)
    visible = np.arange(e_t)[None, :] <= pos[:, None]
    total = np.zeros(e_t, dtype=F64)
    for qh in heads:
        s = scores(q[b, qh, i0:i1, :], k[b, qh // g_size, :e_t, :])
        total += masked_softmax(s, visible).sum(axis=0)
    return total / (len(heads) * (i1 - i0))


def anchor_select_decode_mode(q: np.ndarray, k: np.ndarray, frac_num: int, frac_den: int, mode: str):
    """Anchor decode selection in a head-selection mode: idx
    [B, problems, kk] (ascending) and pooled [B, problems, N]."""
    bsz, n_ctx = k.shape[0], k.shape[2]
    groups = selection_heads(q.shape[1], k.shape[1], mode)
    kk = topk_count(n_ctx, frac_num, frac_den)
    idx = np.zeros((bsz, len(groups), kk), dtype=np.int64)
    pooled = np.zeros((bsz, len(groups), n_ctx), dtype=F64)
    for b in range(bsz):
        for p, heads in enumerate(groups):
            pooled[b, p] = pooled_decode_heads(q, k, b, heads)
            idx[b, p] = select_topk(pooled[b, p], kk)
    return idx, pooled


def anchor_select_prefill_tile_mode(q, k, b, p, t, tile, frac_num, frac_den, mode):
    """Anchor prefill in a head-selection mode, problem p of batch row b and
    tile t: (ascending idx of k_t keys, pooled)."""
    heads = selection_heads(q.shape[1], k.shape[1], mode)[p]
    pooled = pooled_prefill_tile_heads(q, k, b, heads, t, tile)
    return select_topk(pooled, topk_count(pooled.shape[0], frac_num, frac_den)), pooled


def _list_of_head(qh: int, hq: int, hkv: int, mode: str, head_map) -> int:
    """Which anchor list query head qh reads in a reuse (or anchor) layer."""
    g_size = hq // hkv
    if mode == "all":
        return 0
    own = qh if mode == "head" else qh // g_size
    return own if head_map is None else int(head_map[own])


def sparse_decode_mode(q, k, v, idx, mode, head_map=None):
    """Decode attention in a head-selection mode: query head qh attends over
    list idx[b, L(qh)] of its own kv head's keys, L(qh) = head_map[qh // G]
    (gqa), head_map[qh] (head) or 0 (all); head_map None = identity."""
    bsz, hq, _, d = q.shape
    hkv = k.shape[1]
    g_size = hq // hkv
    o = np.zeros((bsz, hq, d), dtype=F64)
    lse = np.zeros((bsz, hq), dtype=F64)
    for b in range(bsz):
        for qh in range(hq):
            sel = np.asarray(idx[b, _list_of_head(qh, hq, hkv, mode, head_map)], dtype=np.int64)
            h = qh // g_size
            vis = np.ones((1, sel.shape[0]), dtype=bool)
            ob, lb = sparse_attend(q[b, qh, 0:1, :], k[b, h, sel], v[b, h, sel], vis)
            o[b, qh], lse[b, qh] = ob[0], lb[0]
    return o, lse


def sparse_prefill_tile_mode(q, k, v, lists, b, t, tile, mode, head_map=None):
    """Prefill attention of query tile t in a head-selection mode: query
    head qh's rows i attend over the keys j <= i of list
    lists[L(qh)] (L as in sparse_decode_mode; lists[p] is tile t's list of
    problem p of batch row b).  Returns o [Hq, rows_t, d], lse [Hq, rows_t]."""
    hq, hkv, n_ctx = q.shape[1], k.shape[1], k.shape[2]
    g_size = hq // hkv
    i0 = t * tile
    i1 = min(i0 + tile, n_ctx)
    pos = np.arange(i0, i1)
    o = np.zeros((hq, i1 - i0, q.shape[-1]), dtype=F64)
    lse = np.zeros((hq, i1 - i0), dtype=F64)
    for qh in range(hq):
        sel = np.asarray(lists[_list_of_head(qh, hq, hkv, mode, head_map)], dtype=np.int64)
        h = qh // g_size
        vis = sel[None, :] <= pos[:, None]
        o[qh], lse[qh] = sparse_attend(q[b, qh, i0:i1, :], k[b, h, sel], v[b, h, sel], vis)
    return o, lse


# ---------------------------------------------------------------------------
# proposal-refine reuse (decode)
#
# The Prism Attention page (abstract; the captions of Figures 2 and 3 and of
# Table 9) replaces rigid reuse with a coarse-to-fine step: a proposal layer
# builds an expanded pool of rho * kappa candidate indices, and each refined
# layer picks its own top-kappa from the pool of its nearest preceding
# proposal layer.  Readings (the page's algorithm listing is not in the text):
# the pool is the proposal layer's own exact Top-(rho kappa) selection, i.e.
# anchor_select_decode with that budget; a refined layer scores only the
# pool's keys, so its post-softmax probabilities are taken over the pool; they
# are pooled over the GQA group as in an anchor layer (head-aware, Kascade
# README Abstract), and the kappa largest win, lowest index on ties, listed
# ascending.  kv head h of the refined layer reads pool head_map[h].


def refine_select_decode(q: np.ndarray, k: np.ndarray, pool, kappa: int, head_map=None):
    """Refined layer: idx [B, Hkv, kappa] (ascending key indices) and the
    pooled scores [B, Hkv, pool_len] of the pool's keys, in pool order."""
    bsz, hq = q.shape[0], q.shape[1]
    hkv = k.shape[1]
    g_size = hq // hkv
    pool = np.asarray(pool, dtype=np.int64)
    n = pool.shape[-1]
    hm = np.arange(hkv) if head_map is None else np.asarray(head_map)
    idx = np.zeros((bsz, hkv, kappa), dtype=np.int64)
    pooled = np.zeros((bsz, hkv, n), dtype=F64)
    for b in range(bsz):
        for h in range(hkv):
            cand = pool[b, hm[h]]
            s = scores(q[b, h * g_size:(h + 1) * g_size, 0, :], k[b, h, cand])
            pooled[b, h] = masked_softmax(s, np.ones_like(s, dtype=bool)).mean(axis=0)
            pos = select_topk(pooled[b, h], kappa)
            idx[b, h] = cand[pos]
    return idx, pooled


# ---------------------------------------------------------------------------
# anchor-layer selection
#
# README, Abstract: the anchor layers are chosen by a dynamic program that
# maximises cross-layer similarity over a development set ("--run_type
# select_layers", Reproducibility, Figure 4).  Readings: the similarity of a
# layer l to an earlier layer a is the overlap of their Top-k index sets,
# |S_a and S_l| / k, averaged over batch rows, lists and tiles (a layer's
# similarity to itself is 1); a plan of M anchors always contains layer 0
# (the first layer has nothing to reuse) and every other layer reuses its
# nearest preceding anchor; the objective is the sum over layers of the
# similarity to the anchor it reuses.  Among equal objectives the plan with
# the lexicographically smallest anchor list wins.


def index_overlap(a, b) -> int:
    """|A and B| for two index lists."""
    return int(np.intersect1d(np.asarray(a), np.asarray(b)).size)


def plan_anchors(sim, n_anchors: int):
    """Best plan for a similarity matrix sim[a][l] (a <= l used): returns
    (anchors ascending, objective).  The recursion: best(m, j) is the best
    objective of layers j.. when layer j is an anchor and m more anchors
    follow it; with none, layers j.. reuse j; otherwise the next anchor i is
    chosen (smallest i among equal objectives)."""
    sim = np.asarray(sim, dtype=F64)
    n = sim.shape[0]
    if not 1 <= n_anchors <= n:
        raise ValueError("need 1 <= anchors <= layers")
    memo = {}

    def best(m, j):
        key = (m, j)
        if key in memo:
            return memo[key]
        if m == 0:
            res = (float(sim[j, j:].sum()), (j,))
        else:
            res = None
            for i in range(j + 1, n - m + 1):
                val, plan = best(m - 1, i)
                tot = float(sim[j, j:i].sum()) + val
                if res is None or tot > res[0]:
                    res = (tot, (j,) + plan)
        memo[key] = res
        return res

    val, plan = best(n_anchors - 1, 0)
    return list(plan), val
