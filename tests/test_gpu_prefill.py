"""GPU parity of the prefill path (score-and-pool + tile Top-k select,
sparse prefill for anchor and reuse layers, dense causal prefill) against
the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from parity import Tally, check_lse, check_out, gen_inputs, np64, prefill_lists

pytestmark = pytest.mark.gpu


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


def _prefill(B, Hq, Hkv, d, N, frac, seed=0, tiles=None, head_map=None, zero_q=False, reuse_seed=None):
    kc = _kc()
    q, k, v = gen_inputs(dict(mode="prefill", B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=seed, zero_q=zero_q)
    s = kc.Shape.make(B, Hq, Hkv, d, N, N, frac)
    ws = kc.Workspace(s)
    idx = kc.select(s, q, k, ws=ws)
    if reuse_seed is not None:
        q, k, v = gen_inputs(dict(mode="prefill", B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=reuse_seed)
    hm = None if head_map is None else torch.tensor(head_map, dtype=torch.int32, device="cuda")
    lse = torch.empty(B, Hq, N, device="cuda")
    o = kc.sparse_prefill(s, q, k, v, idx, hm, lse=lse, ws=ws)
    torch.cuda.synchronize()
    return q, k, v, idx.cpu().numpy(), o, lse


def _judge(q, k, v, idx_flat, o, lse, B, Hkv, N, frac, tiles, head_map=None, sel_inputs=None):
    G = q.shape[1] // Hkv
    rows, off = prefill_lists(idx_flat, B, Hkv, N, frac)
    qs, ks = sel_inputs if sel_inputs is not None else (np64(q), np64(k))
    qn, kn, vn = np64(q), np64(k), np64(v)
    on = np64(o)
    ln = lse.cpu().numpy()
    tally = Tally()
    hm = list(range(Hkv)) if head_map is None else head_map
    for b in range(B):
        for h in range(Hkv):
            for t in tiles:
                sel = rows[b, h, off[t]:off[t + 1]]
                kt = O.topk_count(min(32 * (t + 1), N), *frac)
                assert sel.shape[0] == kt
                pooled = O.pooled_prefill_tile(qs, ks, b, h, t, 32)
                tally.add(O.check_index_set(pooled, kt, sel), (b, h, t))
            for t in tiles:
                sel_h = rows[b, hm[h], off[t]:off[t + 1]]
                o_ref, lse_ref = O.sparse_prefill_tile(qn, kn, vn, sel_h, b, h, t, 32)
                i0, i1 = 32 * t, min(32 * t + 32, N)
                check_out(on[b, h * G:(h + 1) * G, i0:i1], o_ref, f"o b{b} h{h} t{t}")
                check_lse(ln[b, h * G:(h + 1) * G, i0:i1], lse_ref, f"lse b{b} h{h} t{t}")
    tally.assert_ok()
    return tally


@pytest.mark.parametrize("B,Hq,Hkv,d,N,frac", [
    (1, 8, 2, 128, 300, (10, 100)),
    (1, 8, 2, 64, 1000, (10, 100)),
    (2, 8, 8, 128, 257, (20, 100)),      # G = 1
    (1, 16, 2, 128, 400, (5, 100)),      # G = 8
    (1, 4, 1, 64, 1, (10, 100)),         # single key
    (1, 8, 2, 64, 31, (10, 100)),        # one partial tile
    (1, 8, 2, 128, 2100, (1, 1)),        # frac = 1: dense causal
])
def test_prefill_all_tiles(B, Hq, Hkv, d, N, frac):
    q, k, v, idx, o, lse = _prefill(B, Hq, Hkv, d, N, frac, seed=N)
    _judge(q, k, v, idx, o, lse, B, Hkv, N, frac, range(-(-N // 32)))


def test_prefill_reuse_with_head_map():
    B, Hq, Hkv, d, N, frac = 1, 16, 4, 128, 700, (10, 100)
    kc = _kc()
    q0, k0, _ = gen_inputs(dict(mode="prefill", B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=11)
    q, k, v, idx, o, lse = _prefill(B, Hq, Hkv, d, N, frac, seed=11, head_map=[2, 0, 0, 3], reuse_seed=12)
    _judge(q, k, v, idx, o, lse, B, Hkv, N, frac, range(-(-N // 32)), head_map=[2, 0, 0, 3],
           sel_inputs=(np64(q0), np64(k0)))


def test_prefill_zero_query():
    """Q = 0: pooled scores have the closed form of the oracle pin; tiles whose
    k_t does not exceed the keys before them select 0..k_t-1 exactly."""
    B, Hq, Hkv, d, N, frac = 1, 8, 2, 64, 640, (10, 100)
    q, k, v, idx, o, lse = _prefill(B, Hq, Hkv, d, N, frac, zero_q=True)
    rows, off = prefill_lists(idx, B, Hkv, N, frac)
    for t in range(N // 32):
        kt = O.topk_count(32 * (t + 1), *frac)
        if kt <= 32 * t or t == 0:
            assert rows[0, 0, off[t]:off[t + 1]].tolist() == list(range(kt))
    _judge(q, k, v, idx, o, lse, B, Hkv, N, frac, range(N // 32))


def test_dense_prefill_causal():
    kc = _kc()
    B, Hq, Hkv, d, N = 1, 8, 2, 128, 333
    q, k, v = gen_inputs(dict(mode="prefill", B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=9)
    s = kc.Shape.make(B, Hq, Hkv, d, N, N)
    lse = torch.empty(B, Hq, N, device="cuda")
    o = kc.dense_ref(s, q, k, v, causal=True, lse=lse)
    o2 = kc.dense_ref(s, q, k, v, causal=False)
    torch.cuda.synchronize()
    qn, kn, vn = np64(q), np64(k), np64(v)
    for qh in range(Hq):
        ref, lref = O.dense_attention(qn[0, qh], kn[0, qh // 4], vn[0, qh // 4], np.arange(N))
        check_out(np64(o)[0, qh], ref, "dense causal")
        check_lse(lse.cpu().numpy()[0, qh], lref, "dense causal lse")
        ref2, _ = O.dense_attention(qn[0, qh], kn[0, qh // 4], vn[0, qh // 4])
        check_out(np64(o2)[0, qh], ref2, "dense full")


def test_prefill_qwen_stack_sampled():
    """Qwen3-8B-shaped causal prefill (Hq=32, Hkv=8, d=128, N=32768, tile 32):
    anchor layer 0 and reuse layer 1 at full size on the GPU; the oracle
    checks tiles {0, 1, 2, T-1} and 8 seeded random tiles."""
    from sparse_attention_long_anchor_b200 import synth
    kc = _kc()
    cfg = synth.CONFIGS["prefill_qwen8b_n32k"]
    plan, layers = synth.make_stack(cfg, device="cuda", layers=[0, 1])
    frac = (cfg.frac_num, cfg.frac_den)
    s = kc.Shape.make(1, cfg.hq, cfg.hkv, cfg.d, cfg.n_ctx, cfg.n_ctx, frac)
    ws = kc.Workspace(s)
    q0, k0, v0 = layers[0]
    idx = kc.select(s, q0, k0, ws=ws)
    q1, k1, v1 = layers[1]
    hm = plan[1][2]
    lse = torch.empty(1, cfg.hq, cfg.n_ctx, device="cuda")
    o1 = kc.sparse_prefill(s, q1, k1, v1, idx, torch.tensor(hm, dtype=torch.int32, device="cuda"), lse=lse,
                           ws=ws)
    torch.cuda.synchronize()
    T = cfg.n_ctx // 32
    rng = np.random.default_rng(0)
    tiles = sorted(set([0, 1, 2, T - 1] + rng.integers(3, T - 1, size=8).tolist()))
    _judge(q1, k1, v1, idx.cpu().numpy(), o1, lse, 1, cfg.hkv, cfg.n_ctx, frac, tiles, head_map=hm,
           sel_inputs=(np64(q0), np64(k0)))


@pytest.mark.parametrize("Hq,Hkv", [(10, 2), (12, 2), (14, 2)])
def test_prefill_groups_of_five_to_seven(Hq, Hkv):
    """G in {5, 6, 7}: warp-MMA scoring (G > 4) and the warp-MMA sparse
    prefill (the tensor-core kernel takes G <= 4 or multiples of 4)."""
    B, d, N, frac = 1, 128, 330, (10, 100)
    q, k, v, idx, o, lse = _prefill(B, Hq, Hkv, d, N, frac, seed=Hq, head_map=[1, 0], reuse_seed=Hq + 100)
    qs, ks, _ = gen_inputs(dict(mode="prefill", B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=Hq)
    _judge(q, k, v, idx, o, lse, B, Hkv, N, frac, range(-(-N // 32)), head_map=[1, 0],
           sel_inputs=(np64(qs), np64(ks)))
