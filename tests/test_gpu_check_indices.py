"""KASCADE_FLAG_CHECK_INDICES on the GPU: valid inputs give results bit for bit
equal to the unchecked calls with the error word clear; out-of-range list
entries, head_map entries and kv_lens, and lists that are not ascending,
set the word to KASCADE_DEVERR_INDEX_LIST, and the checked call then equals
the unchecked call on the inputs clamped into range.

The K and V tensors of the planted cases are views inside larger buffers
(64 rows of margin on both sides of every tensor), so even a row read at a
planted out-of-range key would stay inside an allocation."""
import pytest
import torch

import oracle as O
from parity import gen_inputs

pytestmark = pytest.mark.gpu

MARGIN_ROWS = 64


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


def _inside(t):
    """A copy of t that is a view into a buffer with margins on both sides."""
    d = t.shape[-1]
    m = MARGIN_ROWS * d
    big = torch.zeros(t.numel() + 2 * m, dtype=t.dtype, device=t.device)
    view = big[m:m + t.numel()].view(t.shape)
    view.copy_(t)
    return view, big


def _decode_case(kc, B=2, Hq=16, Hkv=4, d=128, N=3000, mode=0):
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=N + mode)
    k, kbig = _inside(k)
    v, vbig = _inside(v)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, (10, 100), mode=mode)
    c = s.with_flags(kc.FLAG_CHECK_INDICES)
    ws = kc.Workspace(c, (kc.OP_SELECT, kc.OP_SELECT_VARLEN, kc.OP_SPARSE_DECODE))
    idx = kc.select(s, q, k, ws=ws)
    return q, k, v, s, c, ws, idx, (kbig, vbig)


@pytest.mark.parametrize("mode", [0, 1])
def test_checked_decode_equals_unchecked_on_valid_lists(mode):
    kc = _kc()
    B, Hq, Hkv, d, N = 2, 16, 4, 128, 3000
    q, k, v, s, c, ws, idx, _keep = _decode_case(kc, B, Hq, Hkv, d, N, mode)
    L = s.n_lists
    hm = torch.arange(L, dtype=torch.int32, device="cuda").flip(0).contiguous()
    o0 = kc.sparse_decode(s, q, k, v, idx, hm, ws=ws)
    o1 = kc.sparse_decode(c, q, k, v, idx, hm, ws=ws)
    kvl = torch.tensor([N, N - 777], dtype=torch.int32, device="cuda")
    sel = kc.select_varlen(s, q, k, kvl, ws=ws)
    vl0 = kc.sparse_decode_varlen(s, q, k, v, kvl, sel, hm, ws=ws)
    vl1 = kc.sparse_decode_varlen(c, q, k, v, kvl, sel, hm, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    assert torch.equal(o0, o1)
    assert torch.equal(vl0, vl1)


def test_checked_decode_flags_and_clamps_bad_entries():
    kc = _kc()
    B, Hq, Hkv, d, N = 2, 16, 4, 128, 3000
    q, k, v, s, c, ws, idx, _keep = _decode_case(kc, B, Hq, Hkv, d, N)
    kk = O.topk_count(N, 10, 100)
    lists = idx.view(B, Hkv, kk)
    cases = []
    bad = lists.clone()
    bad[0, 0, 5] = N + 7                 # past the last key
    cases.append(bad)
    bad = lists.clone()
    bad[B - 1, Hkv - 1, kk - 1] = -2     # negative
    cases.append(bad)
    bad = lists.clone()
    bad[1, 2, [3, 4]] = bad[1, 2, [4, 3]]   # in range, not ascending
    cases.append(bad)
    for bad in cases:
        bad = bad.contiguous().view(-1)
        o = kc.sparse_decode(c, q, k, v, bad, None, ws=ws)
        torch.cuda.synchronize()
        assert ws.error(clear=True) == kc.DEVERR_INDEX_LIST
        ref = kc.sparse_decode(s, q, k, v, bad.clamp(0, N - 1).contiguous(), None, ws=ws)
        torch.cuda.synchronize()
        assert ws.error() == 0
        assert torch.equal(o, ref)
    # a head_map entry out of range reads list 0
    hm = torch.tensor([1, 0, Hkv + 3, 2], dtype=torch.int32, device="cuda")
    o = kc.sparse_decode(c, q, k, v, idx, hm, ws=ws)
    torch.cuda.synchronize()
    assert ws.error(clear=True) == kc.DEVERR_INDEX_LIST
    ref = kc.sparse_decode(s, q, k, v, idx, torch.tensor([1, 0, 0, 2], dtype=torch.int32, device="cuda"), ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(o, ref)


def test_checked_varlen_and_paged():
    kc = _kc()
    B, Hq, Hkv, d, N = 2, 16, 4, 128, 3000
    q, k, v, s, c, ws, idx, _keep = _decode_case(kc, B, Hq, Hkv, d, N)
    # kv_lens past N: flagged and clamped to N (the attention reads at most N)
    kvl = torch.tensor([N + 100, N - 5], dtype=torch.int32, device="cuda")
    sel = kc.select_varlen(s, q, k, torch.tensor([N, N - 5], dtype=torch.int32, device="cuda"), ws=ws)
    o = kc.sparse_decode_varlen(c, q, k, v, kvl, sel, None, ws=ws)
    torch.cuda.synchronize()
    assert ws.error(clear=True) == kc.DEVERR_INDEX_LIST
    ref = kc.sparse_decode_varlen(s, q, k, v, torch.tensor([N, N - 5], dtype=torch.int32, device="cuda"), sel,
                                  None, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    assert torch.equal(o, ref)
    # paged cache: identity page table, a list entry past N
    P = 128
    pages = -(-N // P)
    kp = torch.zeros(pages, Hkv, P, d, dtype=k.dtype, device="cuda")
    vp = torch.zeros_like(kp)
    for i in range(pages):              # batch row 0, pages in order
        j0, j1 = i * P, min(N, (i + 1) * P)
        kp[i, :, :j1 - j0] = k[0, :, j0:j1]
        vp[i, :, :j1 - j0] = v[0, :, j0:j1]
    s1 = kc.Shape.make(1, Hq, Hkv, d, 1, N, (10, 100))
    c1 = s1.with_flags(kc.FLAG_CHECK_INDICES)
    pt = torch.arange(pages, dtype=torch.int32, device="cuda").view(1, pages).contiguous()
    kk = O.topk_count(N, 10, 100)
    lst = idx.view(B, Hkv, kk)[:1].clone()
    lst[0, 1, kk // 2] = N + 1     # inside the last page's padding rows, past the keys
    lst = lst.contiguous().view(-1)
    o = kc.sparse_decode_paged(c1, q[:1].contiguous(), kp, vp, pt, P, lst, None, ws=ws)
    torch.cuda.synchronize()
    assert ws.error(clear=True) == kc.DEVERR_INDEX_LIST
    ref = kc.sparse_decode_paged(s1, q[:1].contiguous(), kp, vp, pt, P, lst.clamp(0, N - 1).contiguous(), None,
                                 ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(o, ref)


def test_checked_prefill():
    kc = _kc()
    B, Hq, Hkv, d, N = 1, 8, 2, 128, 300
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N, mode="prefill"), seed=17)
    s = kc.Shape.make(B, Hq, Hkv, d, N, N, (20, 100))
    c = s.with_flags(kc.FLAG_CHECK_INDICES)
    ws = kc.Workspace(c)
    idx = kc.select(s, q, k, ws=ws)
    o0 = kc.sparse_prefill(s, q, k, v, idx, None, ws=ws)
    o1 = kc.sparse_prefill(c, q, k, v, idx, None, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    assert torch.equal(o0, o1)
    # tile 1 (keys [0, 64)) naming key 70: in the context but past the tile's
    # causal end; clamped to 63
    off = O.index_offsets(N, 32, 20, 100)
    row = int(off[-1])
    bad = idx.clone()
    j = int(off[1]) + int(off[2] - off[1]) - 1    # the tile's last entry
    bad[row + j] = 70                              # second list of the row
    o = kc.sparse_prefill(c, q, k, v, bad, None, ws=ws)
    torch.cuda.synchronize()
    assert ws.error(clear=True) == kc.DEVERR_INDEX_LIST
    fixed = bad.clone()
    fixed[row + j] = 63
    ref = kc.sparse_prefill(s, q, k, v, fixed, None, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(o, ref)


def test_checked_refine_pool():
    kc = _kc()
    B, Hq, Hkv, d, N = 1, 8, 2, 128, 4096
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=23)
    k, _kbig = _inside(k)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, (10, 100))
    c = s.with_flags(kc.FLAG_CHECK_INDICES)
    ws = kc.Workspace(c)
    pool_s = kc.Shape.make(B, Hq, Hkv, d, 1, N, (30, 100))
    pool = kc.select(pool_s, q, k, ws=kc.Workspace(pool_s))
    pl = O.topk_count(N, 30, 100)
    r0 = kc.refine_select(s, q, k, pool, pl, ws=ws)
    r1 = kc.refine_select(c, q, k, pool, pl, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    assert torch.equal(r0, r1)
    bad = pool.clone()
    bad[pl - 1] = N + 3                       # last entry of the first pool
    r = kc.refine_select(c, q, k, bad, pl, ws=ws)
    torch.cuda.synchronize()
    assert ws.error(clear=True) == kc.DEVERR_INDEX_LIST
    ref = kc.refine_select(s, q, k, bad.clamp(0, N - 1).contiguous(), pl, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(r, ref)
