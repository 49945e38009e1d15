"""GPU parity of the proposal-refine selection (a refined decode layer picks
its own Top-k from the proposal layer's expanded pool) against the fp64
oracle: index sets by the acceptance rule, judged on the oracle's pooled
values over the pool, and the refined layer's sparse decode."""
import numpy as np
import pytest
import torch

import oracle as O
from parity import Tally, check_out, gen_inputs, np64

pytestmark = pytest.mark.gpu


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


def _judge(qn, kn, pool, got, kappa, hm):
    """Index sets of every (b, h) against the oracle's pool-order values."""
    B, Hkv = got.shape[0], got.shape[1]
    _, pooled = O.refine_select_decode(qn, kn, pool, kappa, hm)
    tally = Tally()
    for b in range(B):
        for h in range(Hkv):
            cand = pool[b, hm[h] if hm is not None else h]
            pos = np.searchsorted(cand, got[b, h])
            assert (pos < len(cand)).all() and (cand[np.minimum(pos, len(cand) - 1)] == got[b, h]).all(), \
                "refined keys must come from the pool"
            tally.add(O.check_index_set(pooled[b, h], kappa, pos), (b, h))
    tally.assert_ok()


@pytest.mark.parametrize("B,Hq,Hkv,d,N,kappa_pct,rho,dtype", [
    (1, 8, 2, 64, 2048, 10, 4, 0),
    (1, 32, 8, 128, 32768, 10, 4, 0),    # the Llama-shaped layer, pool 40 %
    (2, 16, 2, 128, 5000, 5, 2, 0),      # G = 8
    (1, 8, 2, 64, 2048, 10, 4, 1),       # fp32 inputs
])
def test_refine_matches_oracle(B, Hq, Hkv, d, N, kappa_pct, rho, dtype):
    kc = _kc()
    q0, k0, _ = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=N)          # proposal layer
    q1, k1, v1 = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=N + 1)     # refined layer
    if dtype == 1:
        q0, k0, q1, k1, v1 = (t.float().contiguous() for t in (q0, k0, q1, k1, v1))
    prop = kc.Shape.make(B, Hq, Hkv, d, 1, N, (rho * kappa_pct, 100), dtype=dtype)
    pool = kc.select(prop, q0, k0, ws=kc.Workspace(prop))
    pool_len = O.topk_count(N, rho * kappa_pct, 100)
    kappa = O.topk_count(N, kappa_pct, 100)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, (kappa_pct, 100), dtype=dtype)
    hm = list(range(Hkv))[::-1]
    hm_t = torch.tensor(hm, dtype=torch.int32, device="cuda")
    ws = kc.Workspace(s)
    idx = kc.refine_select(s, q1, k1, pool, pool_len, hm_t, ws=ws)
    o = kc.sparse_decode(s, q1, k1, v1, idx, None, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    pool_g = pool.view(B, Hkv, pool_len).cpu().numpy()
    got = idx.view(B, Hkv, kappa).cpu().numpy()
    q1n, k1n, v1n = np64(q1), np64(k1), np64(v1)
    _judge(q1n, k1n, pool_g, got, kappa, hm)
    ref, _ = O.sparse_decode(q1n, k1n, v1n, got)
    if dtype == 1:
        assert np.abs(np64(o).reshape(B, Hq, d) - ref).max() <= 1e-4
    else:
        check_out(np64(o).reshape(B, Hq, d), ref, "refined decode")


def test_refine_edge_pools():
    """A pool of exactly kappa keys comes back unchanged; the whole context
    as the pool gives kascade_select's own sets."""
    kc = _kc()
    B, Hq, Hkv, d, N = 1, 8, 2, 128, 3000
    q, k, _ = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=11)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, (10, 100))
    kappa = O.topk_count(N, 10, 100)
    g = torch.Generator(device="cuda").manual_seed(1)
    small = torch.rand(B * Hkv, N, generator=g, device="cuda").argsort(dim=1)[:, :kappa].sort(dim=1).values
    small = small.to(torch.int32).contiguous()
    got = kc.refine_select(s, q, k, small, kappa)
    whole = torch.arange(N, device="cuda", dtype=torch.int32).repeat(B * Hkv, 1).contiguous()
    got_all = kc.refine_select(s, q, k, whole, N)
    ref = kc.select(s, q, k)
    torch.cuda.synchronize()
    assert torch.equal(got.view(-1), small.view(-1))
    assert torch.equal(got_all, ref)
    # pool lengths outside [kappa, N] are refused before anything runs
    import ctypes
    ws = kc.Workspace(s, (kc.OP_REFINE,))
    for bad in (kappa - 1, N + 1):
        st = kc.lib.kascade_refine_select(ctypes.byref(s), q.data_ptr(), k.data_ptr(), whole.data_ptr(), bad, None,
                                          got.data_ptr(), ws.ptr, ws.nbytes, None)
        assert st == kc.ERR_INVALID_ARG
