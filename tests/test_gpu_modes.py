"""GPU parity of the head-selection variants (per query head, the
oracle_topk strategy; all heads pooled, the head-unaware strategy) against
the fp64 oracle: the index sets by the acceptance rule, and the sparse
attention of anchor and reuse layers on the GPU's own sets."""
import numpy as np
import pytest
import torch

import oracle as O
from parity import Tally, check_lse, check_out, gen_inputs, np64

pytestmark = pytest.mark.gpu

MODE_ID = {"head": 1, "all": 2}


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


def _head_map(mode, Hq, Hkv, seed):
    if mode == "all":
        return None
    n = Hq if mode == "head" else Hkv
    g = np.random.default_rng(seed)
    return g.integers(0, n, n).tolist()


@pytest.mark.parametrize("mode", ["head", "all"])
@pytest.mark.parametrize("B,Hq,Hkv,d,N,frac", [
    (2, 8, 2, 128, 3000, (10, 100)),
    (1, 16, 2, 64, 777, (20, 100)),     # G = 8, ragged N
    (2, 4, 4, 64, 2048, (5, 100)),      # G = 1: every mode pools one head per kv head
])
def test_decode_modes_match_oracle(mode, B, Hq, Hkv, d, N, frac):
    kc = _kc()
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=N + Hq)
    q2, k2, v2 = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=N + Hq + 1)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, frac, mode=MODE_ID[mode])
    ws = kc.Workspace(s)
    idx = kc.select(s, q, k, ws=ws)
    kk = O.topk_count(N, *frac)
    L = s.n_lists
    assert idx.numel() == B * L * kk
    o_a = kc.sparse_decode(s, q, k, v, idx, None, ws=ws)          # anchor: own sets
    hm = _head_map(mode, Hq, Hkv, N)
    hm_t = None if hm is None else torch.tensor(hm, dtype=torch.int32, device="cuda")
    lse = torch.empty(B, Hq, device="cuda")
    o_r = kc.sparse_decode(s, q2, k2, v2, idx, hm_t, lse=lse, ws=ws)   # reuse layer
    torch.cuda.synchronize()
    assert ws.error() == 0
    qn, kn, vn = np64(q), np64(k), np64(v)
    idx_g = idx.view(B, L, kk).cpu().numpy()
    _, pooled = O.anchor_select_decode_mode(qn, kn, *frac, mode)
    tally = Tally()
    for b in range(B):
        for p in range(L):
            tally.add(O.check_index_set(pooled[b, p], kk, idx_g[b, p]), (b, p))
    tally.assert_ok()
    ref_a, _ = O.sparse_decode_mode(qn, kn, vn, idx_g, mode)
    check_out(np64(o_a).reshape(B, Hq, d), ref_a, f"{mode} anchor decode")
    ref_r, lse_r = O.sparse_decode_mode(np64(q2), np64(k2), np64(v2), idx_g, mode, hm)
    check_out(np64(o_r).reshape(B, Hq, d), ref_r, f"{mode} reuse decode")
    check_lse(lse.cpu().numpy(), lse_r, f"{mode} reuse lse")


@pytest.mark.parametrize("mode", ["head", "all"])
@pytest.mark.parametrize("B,Hq,Hkv,d,N,frac", [
    (1, 8, 2, 128, 300, (10, 100)),     # tcgen05 scoring (G = 4), ragged last tile
    (1, 16, 2, 64, 200, (20, 100)),     # warp-MMA scoring (G = 8)
])
def test_prefill_modes_match_oracle(mode, B, Hq, Hkv, d, N, frac):
    kc = _kc()
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N, mode="prefill"), seed=N + 5)
    q2, k2, v2 = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N, mode="prefill"), seed=N + 6)
    s = kc.Shape.make(B, Hq, Hkv, d, N, N, frac, mode=MODE_ID[mode])
    ws = kc.Workspace(s)
    idx = kc.select(s, q, k, ws=ws)
    o_a = kc.sparse_prefill(s, q, k, v, idx, None, ws=ws)
    hm = _head_map(mode, Hq, Hkv, N)
    hm_t = None if hm is None else torch.tensor(hm, dtype=torch.int32, device="cuda")
    lse = torch.empty(B, Hq, N, device="cuda")
    o_r = kc.sparse_prefill(s, q2, k2, v2, idx, hm_t, lse=lse, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    L = s.n_lists
    off = O.index_offsets(N, 32, *frac)
    rows = idx.cpu().numpy().reshape(B, L, int(off[-1]))
    qn, kn, vn = np64(q), np64(k), np64(v)
    q2n, k2n, v2n = np64(q2), np64(k2), np64(v2)
    tally = Tally()
    T = -(-N // 32)
    for b in range(B):
        for t in range(T):
            lists = [rows[b, p, off[t]:off[t + 1]] for p in range(L)]
            for p in range(L):
                _, pooled = O.anchor_select_prefill_tile_mode(qn, kn, b, p, t, 32, *frac, mode)
                tally.add(O.check_index_set(pooled, len(lists[p]), lists[p]), (b, p, t))
            i0, i1 = 32 * t, min(32 * t + 32, N)
            ref_a, _ = O.sparse_prefill_tile_mode(qn, kn, vn, lists, b, t, 32, mode)
            check_out(np64(o_a)[b, :, i0:i1], ref_a, f"{mode} anchor prefill t{t}")
            ref_r, lse_r = O.sparse_prefill_tile_mode(q2n, k2n, v2n, lists, b, t, 32, mode, hm)
            check_out(np64(o_r)[b, :, i0:i1], ref_r, f"{mode} reuse prefill t{t}")
            check_lse(lse.cpu().numpy()[b, :, i0:i1], lse_r, f"{mode} reuse prefill lse t{t}")
    tally.assert_ok()


def test_per_head_decode_many_problems_matches_oracle():
    """Per-head lists over several sequences: 128 problems of one query head
    each (the cluster size follows the problem count)."""
    kc = _kc()
    B, Hq, Hkv, d, N, frac = 4, 32, 8, 128, 32768, (10, 100)
    K = O.topk_count(N, *frac)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, frac, mode=1)
    g = torch.Generator(device="cuda").manual_seed(3)
    q = torch.randn(B, Hq, 1, d, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(B, Hkv, N, d, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(B, Hkv, N, d, generator=g, device="cuda").to(torch.bfloat16)
    idx = torch.rand(B * Hq, N, generator=g, device="cuda").argsort(dim=1)[:, :K].sort(dim=1).values
    idx = idx.to(torch.int32).contiguous()
    hm = torch.randint(0, Hq, (Hq,), generator=g, device="cuda", dtype=torch.int32)
    ws = kc.Workspace(s)
    o = kc.sparse_decode(s, q, k, v, idx, hm, ws=ws)
    o_c = kc.sparse_decode(s, q, k, v, idx, hm)   # without a workspace (no error word)
    torch.cuda.synchronize()
    assert ws.error() == 0
    assert torch.equal(o, o_c)
    # the oracle on the gathered rows of each query head's list
    G = Hq // Hkv
    lists = idx.view(B, Hq, K).long()
    hml = hm.tolist()
    bi = torch.arange(B, device="cuda")[:, None, None]
    kvh = torch.tensor([qh // G for qh in range(Hq)], device="cuda")[None, :, None]
    rows = lists[:, hml, :]
    ks, vs = k[bi, kvh, rows], v[bi, kvh, rows]        # [B, Hq, K, d]
    local = np.tile(np.arange(K), (B, Hq, 1))
    ref, _ = O.sparse_decode_mode(np64(q), np64(ks), np64(vs), local, "head")
    check_out(np64(o).reshape(B, Hq, d), ref, "per-head decode")
