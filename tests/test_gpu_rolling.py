"""Rolling (chunked) prefill: a call whose query rows are the last q_len
positions of the context computes exactly the chunk's tiles of the whole
prompt's prefill (a tile's selection and attention see only the keys up to
its end).  Each chunk is judged against the oracle and against the
whole-prompt call on the same inputs."""
import numpy as np
import pytest
import torch

import oracle as O
from parity import Tally, check_lse, check_out, gen_inputs, np64

pytestmark = pytest.mark.gpu


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


@pytest.mark.parametrize("Hq,Hkv,d,N,frac,dtype", [
    (8, 2, 128, 300, (10, 100), 0),     # tcgen05 kernels
    (16, 2, 64, 200, (20, 100), 0),     # warp-MMA kernels (G = 8)
    (8, 2, 64, 170, (10, 100), 1),      # fp32 inputs
])
def test_rolling_chunks_equal_whole_prefill(Hq, Hkv, d, N, frac, dtype):
    kc = _kc()
    B = 1
    q, k, v = gen_inputs(dict(mode="prefill", B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=N)
    if dtype == 1:
        q, k, v = (t.float().contiguous() for t in (q, k, v))
    full = kc.Shape.make(B, Hq, Hkv, d, N, N, frac, dtype=dtype)
    ws = kc.Workspace(full)
    idx_full = kc.select(full, q, k, ws=ws)
    o_full = kc.sparse_prefill(full, q, k, v, idx_full, None, ws=ws)
    torch.cuda.synchronize()
    off_full = kc.index_offsets(full)
    rows_full = idx_full.cpu().numpy().reshape(B, Hkv, -1)
    qn, kn, vn = np64(q), np64(k), np64(v)
    tol = 1e-4 if dtype == 1 else None
    for c0 in (32, 96, N - N % 32 if N % 32 else N - 32):
        C = N - c0
        qc = q[:, :, c0:].contiguous()
        s = kc.Shape.make(B, Hq, Hkv, d, C, N, frac, dtype=dtype)
        wsc = kc.Workspace(s)
        idx = kc.select(s, qc, k, ws=wsc)
        lse = torch.empty(B, Hq, C, device="cuda")
        o = kc.sparse_prefill(s, qc, k, v, idx, None, lse=lse, ws=wsc)
        od = kc.dense_ref(s, qc, k, v, causal=True)
        torch.cuda.synchronize()
        assert wsc.error() == 0
        t0 = c0 // 32
        off = kc.index_offsets(s)
        assert off.tolist() == (off_full[t0:] - off_full[t0]).tolist()
        rows = idx.cpu().numpy().reshape(B, Hkv, -1)
        on, ln, odn = np64(o), lse.cpu().numpy(), np64(od)
        tally = Tally()
        for h in range(Hkv):
            G = Hq // Hkv
            for i, t in enumerate(range(t0, -(-N // 32))):
                sel = rows[0, h, off[i]:off[i + 1]]
                pooled = O.pooled_prefill_tile(qn, kn, 0, h, t, 32)
                verdict = O.check_index_set(pooled, len(sel), sel)
                tally.add(verdict, (c0, h, t))
                if verdict == "exact":
                    assert (sel == rows_full[0, h, off_full[t]:off_full[t + 1]]).all()
                i0, i1 = 32 * t, min(32 * t + 32, N)
                ref, lref = O.sparse_prefill_tile(qn, kn, vn, sel, 0, h, t, 32)
                got = on[0, h * G:(h + 1) * G, i0 - c0:i1 - c0]
                if tol:
                    assert np.abs(got - ref).max() <= tol
                else:
                    check_out(got, ref, f"chunk {c0} h{h} t{t}")
                    check_lse(ln[0, h * G:(h + 1) * G, i0 - c0:i1 - c0], lref, f"chunk {c0} lse h{h} t{t}")
                for g in range(G):
                    dref, _ = O.dense_attention(qn[0, h * G + g, i0:i1], kn[0, h], vn[0, h],
                                                row_pos=np.arange(i0, i1))
                    if tol:
                        assert np.abs(odn[0, h * G + g, i0 - c0:i1 - c0] - dref).max() <= tol
                    else:
                        check_out(odn[0, h * G + g, i0 - c0:i1 - c0], dref, f"chunk {c0} dense")
        tally.assert_ok()
        if dtype == 0:
            # the chunk's rows of the whole-prompt call, same kernels on the same lists
            check_out(on, np64(o_full)[:, :, c0:], f"chunk {c0} vs whole prompt")


def test_rolling_chunk_shapes_are_checked():
    import ctypes
    kc = _kc()
    bad = kc.Shape.make(1, 8, 2, 64, 100, 300)        # 300 - 100 = 200 is not a multiple of 32
    assert kc.lib.kascade_select(ctypes.byref(bad), 256, 256, 256, None, 0, None) == kc.ERR_UNSUPPORTED
    ok = kc.Shape.make(1, 8, 2, 64, 44, 300)
    assert kc.index_count(ok) == 2 * int(O.index_offsets(300, 32, 10, 100)[-1] - O.index_offsets(300, 32, 10, 100)[8])
