"""GPU parity of the fp32-input variant (q, k, v and o in fp32) against the
fp64 oracle: index sets by the acceptance rule, outputs and log-sum-exp
within 1e-4 absolute on the GPU's own sets (the tolerance stated for fp32
inputs; bf16 rounding alone would exceed it)."""
import numpy as np
import pytest
import torch

import oracle as O
from parity import Tally, gen_inputs, np64

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


def _f32(t, seed):
    """fp32 inputs that are not bf16 values: the synthetic tensors plus
    small fp32 noise."""
    g = torch.Generator(device=t.device).manual_seed(seed)
    return (t.float() + 1e-2 * torch.randn(t.shape, generator=g, device=t.device)).contiguous()


def _close(got, want, what, tol=TOL):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    fin = np.isfinite(want)
    assert np.array_equal(fin, np.isfinite(got)), f"{what}: -inf pattern differs"
    err = np.abs(got[fin] - want[fin]).max() if fin.any() else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e}"


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("B,Hq,Hkv,d,N,frac", [
    (1, 8, 2, 64, 2048, (10, 100)),     # the 2K decode workload's shape
    (2, 16, 2, 128, 1000, (20, 100)),   # G = 8, ragged
])
def test_fp32_decode(mode, B, Hq, Hkv, d, N, frac):
    kc = _kc()
    q, k, v = (_f32(t, i) for i, t in enumerate(gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=N)))
    q2, k2, v2 = (_f32(t, 7 + i) for i, t in enumerate(gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=N + 1)))
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, frac, mode=mode, dtype=kc.DTYPE_F32)
    ws = kc.Workspace(s)
    idx = kc.select(s, q, k, ws=ws)
    kk = O.topk_count(N, *frac)
    L = s.n_lists
    name = O.MODES[mode]
    nmap = {0: Hkv, 1: Hq, 2: 1}[mode]
    hm = np.random.default_rng(N).integers(0, nmap, nmap).tolist() if mode != 2 else None
    hm_t = None if hm is None else torch.tensor(hm, dtype=torch.int32, device="cuda")
    lse_a = torch.empty(B, Hq, device="cuda")
    lse_r = torch.empty(B, Hq, device="cuda")
    o_a = kc.sparse_decode(s, q, k, v, idx, None, lse=lse_a, ws=ws)
    o_r = kc.sparse_decode(s, q2, k2, v2, idx, hm_t, lse=lse_r, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    assert o_a.dtype == torch.float32
    qn, kn, vn = np64(q), np64(k), np64(v)
    idx_g = idx.view(B, L, kk).cpu().numpy()
    _, pooled = O.anchor_select_decode_mode(qn, kn, *frac, name)
    tally = Tally()
    for b in range(B):
        for p in range(L):
            tally.add(O.check_index_set(pooled[b, p], kk, idx_g[b, p]), (b, p))
    tally.assert_ok()
    ref, lref = O.sparse_decode_mode(qn, kn, vn, idx_g, name)
    _close(np64(o_a).reshape(B, Hq, d), ref, "fp32 anchor decode")
    _close(lse_a.cpu().numpy(), lref, "fp32 anchor decode lse")
    ref, lref = O.sparse_decode_mode(np64(q2), np64(k2), np64(v2), idx_g, name, hm)
    _close(np64(o_r).reshape(B, Hq, d), ref, "fp32 reuse decode")
    _close(lse_r.cpu().numpy(), lref, "fp32 reuse decode lse")


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("B,Hq,Hkv,d,N,frac", [
    (1, 8, 2, 128, 300, (10, 100)),
    (1, 16, 2, 64, 160, (20, 100)),     # G = 8
])
def test_fp32_prefill(mode, B, Hq, Hkv, d, N, frac):
    kc = _kc()
    q, k, v = (_f32(t, i) for i, t in
               enumerate(gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N, mode="prefill"), seed=N)))
    s = kc.Shape.make(B, Hq, Hkv, d, N, N, frac, mode=mode, dtype=kc.DTYPE_F32)
    ws = kc.Workspace(s)
    idx = kc.select(s, q, k, ws=ws)
    lse = torch.empty(B, Hq, N, device="cuda")
    o = kc.sparse_prefill(s, q, k, v, idx, None, lse=lse, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    name = O.MODES[mode]
    L = s.n_lists
    off = O.index_offsets(N, 32, *frac)
    rows = idx.cpu().numpy().reshape(B, L, int(off[-1]))
    qn, kn, vn, on, ln = np64(q), np64(k), np64(v), np64(o), lse.cpu().numpy()
    tally = Tally()
    for b in range(B):
        for t in range(-(-N // 32)):
            lists = [rows[b, p, off[t]:off[t + 1]] for p in range(L)]
            for p in range(L):
                _, pooled = O.anchor_select_prefill_tile_mode(qn, kn, b, p, t, 32, *frac, name)
                tally.add(O.check_index_set(pooled, len(lists[p]), lists[p]), (b, p, t))
            i0, i1 = 32 * t, min(32 * t + 32, N)
            ref, lref = O.sparse_prefill_tile_mode(qn, kn, vn, lists, b, t, 32, name)
            _close(on[b, :, i0:i1], ref, f"fp32 prefill t{t}")
            _close(ln[b, :, i0:i1], lref, f"fp32 prefill lse t{t}")
    tally.assert_ok()


def test_fp32_dense():
    kc = _kc()
    B, Hq, Hkv, d, N = 1, 8, 2, 128, 700
    G = Hq // Hkv
    q, k, v = (_f32(t, i) for i, t in enumerate(gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=3)))
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, dtype=kc.DTYPE_F32)
    o = kc.dense_ref(s, q, k, v, causal=False)
    qp, kp, vp = (_f32(t, 5 + i) for i, t in
                  enumerate(gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N, mode="prefill"), seed=4)))
    sp = kc.Shape.make(B, Hq, Hkv, d, N, N, dtype=kc.DTYPE_F32)
    op = kc.dense_ref(sp, qp, kp, vp, causal=True)
    torch.cuda.synchronize()
    qn, kn, vn = np64(q), np64(k), np64(v)
    for h in range(Hkv):
        ref, _ = O.dense_attention(qn[0, h * G:(h + 1) * G, 0], kn[0, h], vn[0, h])
        _close(np64(o)[0, h * G:(h + 1) * G, 0], ref, "fp32 dense decode")
    qn, kn, vn = np64(qp), np64(kp), np64(vp)
    for qh in range(Hq):
        ref, _ = O.dense_attention(qn[0, qh], kn[0, qh // G], vn[0, qh // G], row_pos=np.arange(N))
        _close(np64(op)[0, qh], ref, "fp32 causal dense prefill")


@pytest.mark.parametrize("prefill", [False, True])
def test_fp16_inputs(prefill):
    """fp16 q, k, v (the README kernels' input type): exact index sets and
    outputs, rounded once to fp16, within the bf16 path's tolerances."""
    from parity import check_out
    kc = _kc()
    B, Hq, Hkv, d, N, frac = 1, 8, 2, 128, (300 if prefill else 2048), (10, 100)
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N, mode="prefill" if prefill else "decode")
    q, k, v = (t.half().contiguous() for t in gen_inputs(kw, seed=N + 2))
    s = kc.Shape.make(B, Hq, Hkv, d, N if prefill else 1, N, frac, dtype=kc.DTYPE_F16)
    ws = kc.Workspace(s)
    idx = kc.select(s, q, k, ws=ws)
    o = (kc.sparse_prefill if prefill else kc.sparse_decode)(s, q, k, v, idx, None, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0 and o.dtype == torch.float16
    qn, kn, vn, on = np64(q), np64(k), np64(v), np64(o)
    G = Hq // Hkv
    tally = Tally()
    if prefill:
        off = O.index_offsets(N, 32, *frac)
        rows = idx.cpu().numpy().reshape(B, Hkv, int(off[-1]))
        for h in range(Hkv):
            for t in range(-(-N // 32)):
                sel = rows[0, h, off[t]:off[t + 1]]
                tally.add(O.check_index_set(O.pooled_prefill_tile(qn, kn, 0, h, t, 32), len(sel), sel), (h, t))
                ref, _ = O.sparse_prefill_tile(qn, kn, vn, sel, 0, h, t, 32)
                check_out(on[0, h * G:(h + 1) * G, 32 * t:min(32 * t + 32, N)], ref, f"fp16 prefill h{h} t{t}")
    else:
        kk = O.topk_count(N, *frac)
        idx_g = idx.view(B, Hkv, kk).cpu().numpy()
        _, pooled = O.anchor_select_decode(qn, kn, *frac)
        for h in range(Hkv):
            tally.add(O.check_index_set(pooled[0, h], kk, idx_g[0, h]), h)
        ref, _ = O.sparse_decode(qn, kn, vn, idx_g)
        check_out(on.reshape(B, Hq, d), ref, "fp16 decode")
    tally.assert_ok()
