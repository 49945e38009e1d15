"""Sparse decode over a paged KV cache: the same keys stored in fixed-size
pages named by a per-sequence page table give the contiguous cache's
results bit for bit, and match the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from parity import check_out, gen_inputs, np64

pytestmark = pytest.mark.gpu


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


def _paged(k, v, page_size, seed):
    """Scatter [B, Hkv, N, d] into pages [num_pages, Hkv, P, d] in a shuffled
    order (plus unused pages), and the page table [B, max_pages]."""
    B, Hkv, N, d = k.shape
    per = -(-N // page_size)
    num = B * per + 3
    g = torch.Generator().manual_seed(seed)
    order = torch.randperm(num, generator=g)[:B * per].view(B, per)
    kp = torch.zeros(num, Hkv, page_size, d, dtype=k.dtype, device=k.device)
    vp = torch.zeros_like(kp)
    for b in range(B):
        for i in range(per):
            j0, j1 = i * page_size, min(N, (i + 1) * page_size)
            kp[order[b, i], :, :j1 - j0] = k[b, :, j0:j1]
            vp[order[b, i], :, :j1 - j0] = v[b, :, j0:j1]
    return kp, vp, order.to(torch.int32).to(k.device).contiguous()


@pytest.mark.parametrize("B,Hq,Hkv,d,N,page", [
    (2, 32, 8, 128, 5000, 64),
    (1, 8, 2, 64, 2048, 256),
    (8, 32, 8, 128, 65536, 128),     # the batched 64K decode: 4-CTA clusters, refilled slabs
])
def test_paged_decode_equals_contiguous(B, Hq, Hkv, d, N, page):
    kc = _kc()
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=N + page)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, (10, 100))
    ws = kc.Workspace(s)
    idx = kc.select(s, q, k, ws=ws)
    hm = torch.tensor(list(range(Hkv))[::-1], dtype=torch.int32, device="cuda")
    kp, vp, pt = _paged(k, v, page, seed=N)
    o_c = kc.sparse_decode(s, q, k, v, idx, hm, ws=ws)
    o_p = kc.sparse_decode_paged(s, q, kp, vp, pt, page, idx, hm, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    assert torch.equal(o_c, o_p)
    if N <= 8192:
        kk = O.topk_count(N, 10, 100)
        idx_g = idx.view(B, Hkv, kk).cpu().numpy()
        ref, _ = O.sparse_decode(np64(q), np64(k), np64(v), idx_g, hm.tolist())
        check_out(np64(o_p).reshape(B, Hq, d), ref, "paged decode")
        # dense decode over the paged cache
        od_c = kc.dense_ref(s, q, k, v, causal=False)
        od_p = kc.sparse_decode_paged(s, q, kp, vp, pt, page, None)
        torch.cuda.synchronize()
        assert torch.equal(od_c, od_p)


def test_paged_arguments_are_checked():
    kc = _kc()
    s = kc.Shape.make(1, 8, 2, 64, 1, 1000)
    L = kc.lib
    for page, pages, want in ((48, 30, kc.ERR_UNSUPPORTED), (8, 200, kc.ERR_UNSUPPORTED), (64, 15, kc.ERR_INVALID_ARG)):
        st = L.kascade_sparse_decode_paged(ctypes.byref(s), 256, 256, 256, 256, page, pages, 256, None, 256, None,
                                           None, 0, None)
        assert st == want
