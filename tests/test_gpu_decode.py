"""GPU parity of the decode path (anchor scoring + Top-k select, sparse
decode for anchor and reuse layers, dense decode) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from parity import check_lse, check_out, decode_idx_check, gen_inputs, np64

pytestmark = pytest.mark.gpu


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


def _run_decode(B, Hq, Hkv, d, N, frac, seed=0, zero_q=False, head_map=None, n_salient=64):
    kc = _kc()
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=seed, zero_q=zero_q, n_salient=n_salient)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, frac)
    ws = kc.Workspace(s)
    idx = kc.select(s, q, k, ws=ws)
    kk = O.topk_count(N, *frac)
    hm = None if head_map is None else torch.tensor(head_map, dtype=torch.int32, device="cuda")
    lse = torch.empty(B, Hq, device="cuda")
    o = kc.sparse_decode(s, q, k, v, idx, hm, lse=lse, ws=ws)
    torch.cuda.synchronize()
    qn, kn, vn = np64(q), np64(k), np64(v)
    idx_g = idx.view(B, Hkv, kk).cpu().numpy()
    _, tally = decode_idx_check(qn, kn, idx_g, frac)
    tally.assert_ok()
    o_ref, lse_ref = O.sparse_decode(qn, kn, vn, idx_g, head_map)
    check_out(np64(o).reshape(B, Hq, d), o_ref, "sparse decode")
    check_lse(lse.cpu().numpy(), lse_ref, "sparse decode lse")
    assert ws.error() == 0
    return q, k, v, idx_g, tally


def test_decode_small_config():
    """B=1, Hq=8, Hkv=2 (GQA 4), d=64, N=2048, frac=0.1: anchor + identity reuse."""
    _, _, _, idx_g, tally = _run_decode(1, 8, 2, 64, 2048, (10, 100))
    assert idx_g.shape == (1, 2, 205)


@pytest.mark.parametrize("B,Hq,Hkv,d,N,frac", [
    (1, 8, 2, 128, 2048, (10, 100)),
    (2, 8, 8, 64, 1000, (10, 100)),       # G = 1
    (2, 16, 2, 128, 777, (5, 100)),       # G = 8, ragged N
    (1, 4, 1, 64, 1, (10, 100)),          # single key
    (1, 8, 2, 64, 33, (1, 100)),          # tiny k
    (3, 8, 2, 128, 4095, (20, 100)),
    (1, 8, 2, 64, 300, (1, 1)),           # frac = 1: everything selected
])
def test_decode_sweep(B, Hq, Hkv, d, N, frac):
    _run_decode(B, Hq, Hkv, d, N, frac, seed=B * 7 + N)


def test_decode_reuse_head_map():
    kc = _kc()
    B, Hq, Hkv, d, N, frac = 2, 16, 4, 128, 3000, (10, 100)
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=3)
    q2, k2, v2 = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=4)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, frac)
    ws = kc.Workspace(s)
    idx = kc.select(s, q, k, ws=ws)
    head_map = [3, 3, 0, 1]
    hm = torch.tensor(head_map, dtype=torch.int32, device="cuda")
    lse = torch.empty(B, Hq, device="cuda")
    o = kc.sparse_decode(s, q2, k2, v2, idx, hm, lse=lse, ws=ws)
    torch.cuda.synchronize()
    kk = O.topk_count(N, *frac)
    idx_g = idx.view(B, Hkv, kk).cpu().numpy()
    o_ref, lse_ref = O.sparse_decode(np64(q2), np64(k2), np64(v2), idx_g, head_map)
    check_out(np64(o).reshape(B, Hq, d), o_ref, "reuse decode")
    check_lse(lse.cpu().numpy(), lse_ref, "reuse lse")
    # a second call gives the identical result
    o2 = kc.sparse_decode(s, q2, k2, v2, idx, hm, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(o, o2)


def test_decode_zero_query_ties_go_to_lowest_index():
    """Q = 0: all pooled scores tie, so the lowest k indices must win and the
    output is the mean of V over them."""
    B, Hq, Hkv, d, N, frac = 1, 8, 2, 64, 2048, (10, 100)
    q, k, v, idx_g, _ = _run_decode(B, Hq, Hkv, d, N, frac, zero_q=True)
    kk = O.topk_count(N, *frac)
    assert np.array_equal(idx_g[0, 0], np.arange(kk)) and np.array_equal(idx_g[0, 1], np.arange(kk))


@pytest.mark.parametrize("B,Hq,Hkv,d,N", [
    (2, 16, 4, 128, 5000),     # long lists: contiguous rows as whole 16-row tiles, ragged tail
    (1, 8, 2, 64, 9001),       # d = 64: one tile per row block
    (1, 32, 8, 128, 32768),    # the Llama-shaped layer, the dense denominator of the benchmark
    (1, 8, 2, 128, 700),       # short lists: the up-front form
])
def test_dense_decode(B, Hq, Hkv, d, N):
    kc = _kc()
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=5 + N)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N)
    lse = torch.empty(B, Hq, device="cuda")
    o = kc.dense_ref(s, q, k, v, lse=lse, ws=kc.Workspace(s, (kc.OP_DENSE,)))
    torch.cuda.synchronize()
    qn, kn, vn = np64(q), np64(k), np64(v)
    all_idx = np.broadcast_to(np.arange(N), (B, Hkv, N))
    o_ref, lse_ref = O.sparse_decode(qn, kn, vn, all_idx)
    check_out(np64(o).reshape(B, Hq, d), o_ref, "dense decode")
    check_lse(lse.cpu().numpy(), lse_ref, "dense decode lse")


def test_decode_llama_stack_layers():
    """The 32-layer Llama-shaped stack (B=1, Hq=32, Hkv=8, d=128, N=32768):
    anchor layer 0 (full check of all 8 index sets) and reuse layer 1 with its
    random head_map, in the launch configuration the benchmark uses."""
    from sparse_attention_long_anchor_b200 import synth
    kc = _kc()
    cfg = synth.CONFIGS["decode_llama8b_n32k"]
    plan, layers = synth.make_stack(cfg, device="cuda", layers=[0, 1])
    s = kc.Shape.make(cfg.batch, cfg.hq, cfg.hkv, cfg.d, 1, cfg.n_ctx, (cfg.frac_num, cfg.frac_den))
    ws = kc.Workspace(s)
    q0, k0, v0 = layers[0]
    idx = kc.select(s, q0, k0, ws=ws)
    o0 = kc.sparse_decode(s, q0, k0, v0, idx, None, ws=ws)
    q1, k1, v1 = layers[1]
    hm = plan[1][2]
    o1 = kc.sparse_decode(s, q1, k1, v1, idx, torch.tensor(hm, dtype=torch.int32, device="cuda"), ws=ws)
    torch.cuda.synchronize()
    kk = O.topk_count(cfg.n_ctx, cfg.frac_num, cfg.frac_den)
    idx_g = idx.view(1, cfg.hkv, kk).cpu().numpy()
    qn, kn, vn = np64(q0), np64(k0), np64(v0)
    _, tally = decode_idx_check(qn, kn, idx_g, (cfg.frac_num, cfg.frac_den))
    tally.assert_ok()
    o_ref, _ = O.sparse_decode(qn, kn, vn, idx_g)
    check_out(np64(o0).reshape(1, cfg.hq, cfg.d), o_ref, "anchor layer")
    o_ref1, _ = O.sparse_decode(np64(q1), np64(k1), np64(v1), idx_g, hm)
    check_out(np64(o1).reshape(1, cfg.hq, cfg.d), o_ref1, "reuse layer")


def test_decode_pdl_flags_give_identical_results():
    """Programmatic dependent launch (and early gathers for inputs written two
    launches back) changes scheduling only, never results."""
    kc = _kc()
    B, Hq, Hkv, d, N, frac = 1, 32, 8, 128, 8192, (10, 100)
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=21)
    q2, k2, v2 = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=22)
    hm = torch.tensor([1, 0, 3, 2, 5, 4, 7, 6], dtype=torch.int32, device="cuda")
    outs = []
    for flags in (0, kc.FLAG_PDL, kc.FLAG_PDL | kc.FLAG_INPUTS_STABLE):
        s = kc.Shape.make(B, Hq, Hkv, d, 1, N, frac, flags=flags & kc.FLAG_PDL)
        ws = kc.Workspace(s)
        idx = kc.select(s, q, k, ws=ws)
        o0 = kc.sparse_decode(s, q, k, v, idx, None, ws=ws)
        o1 = kc.sparse_decode(s.with_flags(flags), q2, k2, v2, idx, hm, ws=ws)
        o2 = kc.sparse_decode(s.with_flags(flags), q, k2, v2, idx, hm, ws=ws)
        torch.cuda.synchronize()
        assert ws.error() == 0
        outs.append((idx.clone(), o0.clone(), o1.clone(), o2.clone()))
    for other in outs[1:]:
        for x, y in zip(outs[0], other):
            assert torch.equal(x, y)


def test_decode_long_context_takes_the_two_kernel_path():
    """A context whose scores do not fit on chip (N = 131072, G = 4) runs the
    scoring kernel plus the 8-CTA cluster select; the Llama-shaped anchor
    (N = 32768) runs the fused single launch.  Both match the oracle."""
    kc = _kc()
    B, Hq, Hkv, d, N, frac = 1, 8, 2, 128, 131072, (10, 100)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, frac)
    assert kc.launch_count(s, kc.OP_SELECT) == 2
    assert kc.launch_count(kc.Shape.make(1, 32, 8, 128, 1, 32768, frac), kc.OP_SELECT) == 1
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=31)
    ws = kc.Workspace(s)
    idx = kc.select(s, q, k, ws=ws)
    o = kc.sparse_decode(s, q, k, v, idx, None, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    kk = O.topk_count(N, *frac)
    idx_g = idx.view(B, Hkv, kk).cpu().numpy()
    qn, kn, vn = np64(q), np64(k), np64(v)
    _, tally = decode_idx_check(qn, kn, idx_g, frac)
    tally.assert_ok()
    o_ref, _ = O.sparse_decode(qn, kn, vn, idx_g)
    check_out(np64(o).reshape(B, Hq, d), o_ref, "long-context decode")


def test_decode_beyond_the_cluster_select_range():
    """N > 131072 (the 8-CTA cluster select holds up to 16384 keys per CTA):
    scoring kernel plus the one-CTA-per-problem Top-k, up to the largest
    context the library accepts."""
    kc = _kc()
    for N, seed in ((200003, 41), (1 << 20, 42)):
        B, Hq, Hkv, d, frac = 1, 4, 1, 64, (10, 100)
        s = kc.Shape.make(B, Hq, Hkv, d, 1, N, frac)
        assert kc.launch_count(s, kc.OP_SELECT) == 2
        q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=seed)
        ws = kc.Workspace(s)
        idx = kc.select(s, q, k, ws=ws)
        o = kc.sparse_decode(s, q, k, v, idx, None, ws=ws)
        torch.cuda.synchronize()
        assert ws.error() == 0
        kk = O.topk_count(N, *frac)
        idx_g = idx.view(B, Hkv, kk).cpu().numpy()
        qn, kn, vn = np64(q), np64(k), np64(v)
        _, tally = decode_idx_check(qn, kn, idx_g, frac)
        tally.assert_ok()
        o_ref, _ = O.sparse_decode(qn, kn, vn, idx_g)
        check_out(np64(o).reshape(B, Hq, d), o_ref, f"decode N={N}")
