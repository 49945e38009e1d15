"""GPU parity at the largest workloads, on sampled problems.

* Batched decode, Llama-shaped (B=8, Hq=32, Hkv=8, d=128, N=65536, 10 %):
  anchor layer 0 and reuse layer 1 run in full on the GPU; the oracle judges
  every kv head of batches {0, 3, 7}.
* Long causal prefill (Hq=32, Hkv=8, d=128, N=131072, tile 32) at
  frac 5 %, 10 % and 20 %: anchor layer 0 selects, reuse layer 1 attends;
  the oracle judges tiles {0, 1, 2, T-1} plus seeded random tiles on every
  kv head.

Host copies are fp32 (bf16 widens exactly); the oracle widens each slice it
reads to fp64.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity import Tally, check_lse, check_out, prefill_lists

pytestmark = pytest.mark.gpu


def _f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def test_decode_batched_b8_n64k_sampled():
    from sparse_attention_long_anchor_b200 import kascade as kc, synth
    cfg = synth.CONFIGS["decode_llama8b_b8_n64k"]
    plan, layers = synth.make_stack(cfg, device="cuda", layers=[0, 1])
    frac = (cfg.frac_num, cfg.frac_den)
    s = kc.Shape.make(cfg.batch, cfg.hq, cfg.hkv, cfg.d, 1, cfg.n_ctx, frac)
    ws = kc.Workspace(s)
    q0, k0, v0 = layers[0]
    idx = kc.select(s, q0, k0, ws=ws)
    flags = kc.FLAG_PDL
    o0 = kc.sparse_decode(s.with_flags(flags), q0, k0, v0, idx, None, ws=ws)
    q1, k1, v1 = layers[1]
    hm = plan[1][2]
    o1 = kc.sparse_decode(s.with_flags(flags | kc.FLAG_INPUTS_STABLE), q1, k1, v1, idx,
                          torch.tensor(hm, dtype=torch.int32, device="cuda"), ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    kk = O.topk_count(cfg.n_ctx, *frac)
    idx_g = idx.view(cfg.batch, cfg.hkv, kk).cpu().numpy()
    tally = Tally()
    for b in (0, 3, cfg.batch - 1):
        qb, kb = _f32(q0[b:b + 1]), _f32(k0[b:b + 1])
        _, pooled = O.anchor_select_decode(qb, kb, *frac)
        for h in range(cfg.hkv):
            tally.add(O.check_index_set(pooled[0, h], kk, idx_g[b, h]), (b, h))
        o_ref, _ = O.sparse_decode(qb, kb, _f32(v0[b:b + 1]), idx_g[b:b + 1])
        check_out(_f32(o0[b:b + 1]).reshape(1, cfg.hq, cfg.d), o_ref, f"anchor b{b}")
        o_ref1, _ = O.sparse_decode(_f32(q1[b:b + 1]), _f32(k1[b:b + 1]), _f32(v1[b:b + 1]),
                                    idx_g[b:b + 1], hm)
        check_out(_f32(o1[b:b + 1]).reshape(1, cfg.hq, cfg.d), o_ref1, f"reuse b{b}")
    tally.assert_ok()


@pytest.mark.parametrize("frac_num", [5, 10, 20])
def test_prefill_long_128k_sampled(frac_num):
    from sparse_attention_long_anchor_b200 import kascade as kc, synth
    cfg = synth.CONFIGS["prefill_n128k"].with_(frac_num=frac_num)
    plan, layers = synth.make_stack(cfg, device="cuda", layers=[0, 1])
    frac = (cfg.frac_num, cfg.frac_den)
    N = cfg.n_ctx
    s = kc.Shape.make(1, cfg.hq, cfg.hkv, cfg.d, N, N, frac)
    ws = kc.Workspace(s)
    q0, k0, _ = layers[0]
    idx = kc.select(s.with_flags(kc.FLAG_PDL), q0, k0, ws=ws)
    q1, k1, v1 = layers[1]
    hm = plan[1][2]
    lse = torch.empty(1, cfg.hq, N, device="cuda")
    o1 = kc.sparse_prefill(s.with_flags(kc.FLAG_PDL), q1, k1, v1, idx,
                           torch.tensor(hm, dtype=torch.int32, device="cuda"), lse=lse, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    T = N // 32
    rng = np.random.default_rng(frac_num)
    tiles = sorted(set([0, 1, 2, T - 1] + rng.integers(3, T - 1, size=4).tolist()))
    G = cfg.hq // cfg.hkv
    rows, off = prefill_lists(idx.cpu().numpy(), 1, cfg.hkv, N, frac)
    qs, ks = _f32(q0), _f32(k0)
    qn, kn, vn = _f32(q1), _f32(k1), _f32(v1)
    on, ln = _f32(o1), lse.cpu().numpy()
    tally = Tally()
    for h in range(cfg.hkv):
        for t in tiles:
            sel = rows[0, h, off[t]:off[t + 1]]
            kt = O.topk_count(min(32 * (t + 1), N), *frac)
            assert sel.shape[0] == kt
            pooled = O.pooled_prefill_tile(qs, ks, 0, h, t, 32)
            tally.add(O.check_index_set(pooled, kt, sel), (h, t))
            sel_h = rows[0, hm[h], off[t]:off[t + 1]]
            o_ref, lse_ref = O.sparse_prefill_tile(qn, kn, vn, sel_h, 0, h, t, 32)
            i0, i1 = 32 * t, min(32 * t + 32, N)
            check_out(on[0, h * G:(h + 1) * G, i0:i1], o_ref, f"o h{h} t{t}")
            check_lse(ln[0, h * G:(h + 1) * G, i0:i1], lse_ref, f"lse h{h} t{t}")
    tally.assert_ok()
