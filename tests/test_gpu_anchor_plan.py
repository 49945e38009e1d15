"""Anchor-layer selection on the GPU: the index-set overlap kernel against
exact set intersections of the same lists, and a plan from the overlaps of
a synthetic stack's per-layer selections, native planner against the
oracle's recursion."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


def test_overlap_counts_and_plan_on_a_decode_stack():
    from sparse_attention_long_anchor_b200 import synth
    kc = _kc()
    cfg = synth.CONFIGS["decode_b1_h8_n2k"].with_(n_layers=8, anchors=(0,), head_map="random", drift=True, batch=2)
    plan, layers = synth.make_stack(cfg, device="cuda")
    s = kc.Shape.make(cfg.batch, cfg.hq, cfg.hkv, cfg.d, 1, cfg.n_ctx, (cfg.frac_num, cfg.frac_den))
    ws = kc.Workspace(s)
    idx = [kc.select(s, layers[l][0], layers[l][1], ws=ws).clone() for l in range(cfg.n_layers)]
    kk = O.topk_count(cfg.n_ctx, cfg.frac_num, cfg.frac_den)
    L = cfg.n_layers
    sim = np.zeros((L, L))
    host = [t.view(cfg.batch, cfg.hkv, kk).cpu().numpy() for t in idx]
    for a in range(L):
        for l in range(a, L):
            counts = kc.index_overlap(s, idx[a], idx[l])
            torch.cuda.synchronize()
            got = counts.cpu().numpy().reshape(cfg.batch, cfg.hkv)
            for b in range(cfg.batch):
                for h in range(cfg.hkv):
                    assert got[b, h] == O.index_overlap(host[a][b, h], host[l][b, h])
            sim[a, l] = got.mean() / kk
    assert np.allclose(np.diag(sim), 1.0)
    for m in (1, 2, 3, 4):
        got_plan = kc.plan_anchors(sim, m)
        want_plan = O.plan_anchors(sim, m)
        assert got_plan[0] == want_plan[0] and abs(got_plan[1] - want_plan[1]) < 1e-9


def test_overlap_counts_prefill_tiles():
    from parity import gen_inputs
    kc = _kc()
    B, Hq, Hkv, d, N = 1, 8, 2, 64, 200
    s = kc.Shape.make(B, Hq, Hkv, d, N, N, (20, 100))
    qa, ka, _ = gen_inputs(dict(mode="prefill", B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=1)
    qb, kb, _ = gen_inputs(dict(mode="prefill", B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=2)
    ia, ib = kc.select(s, qa, ka), kc.select(s, qb, kb)
    counts = kc.index_overlap(s, ia, ib)
    torch.cuda.synchronize()
    off = O.index_offsets(N, 32, 20, 100)
    ra = ia.cpu().numpy().reshape(B, Hkv, -1)
    rb = ib.cpu().numpy().reshape(B, Hkv, -1)
    for h in range(Hkv):
        want = sum(O.index_overlap(ra[0, h, off[t]:off[t + 1]], rb[0, h, off[t]:off[t + 1]])
                   for t in range(len(off) - 1))
        assert counts[h].item() == want
    same = kc.index_overlap(s, ia, ia)
    torch.cuda.synchronize()
    assert (same.cpu().numpy() == off[-1]).all()
