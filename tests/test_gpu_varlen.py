"""Variable-length decode batches: each batch row selects and attends as a
batch of one with its own context length; lists keep the layout of the
longest context and end in -1."""
import numpy as np
import pytest
import torch

import oracle as O
from parity import Tally, check_lse, check_out, gen_inputs, np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Hq,Hkv,d,N,lens,mode", [
    (8, 2, 128, 4000, [4000, 1500, 33], 0),
    (16, 2, 64, 2500, [1, 2500, 700, 1999], 0),    # G = 8, a one-key row
    (8, 2, 64, 3000, [3000, 1200], 1),             # per-head lists
])
def test_varlen_decode_matches_per_row_oracle(Hq, Hkv, d, N, lens, mode):
    from sparse_attention_long_anchor_b200 import kascade as kc
    B = len(lens)
    frac = (10, 100)
    q, k, v = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=N + B)
    kv = torch.tensor(lens, dtype=torch.int32, device="cuda")
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, frac, mode=mode)
    idx = kc.select_varlen(s, q, k, kv)
    hm = None if mode != 0 else torch.tensor(list(range(Hkv))[::-1], dtype=torch.int32, device="cuda")
    lse = torch.empty(B, Hq, device="cuda")
    o = kc.sparse_decode_varlen(s, q, k, v, kv, idx, hm, lse=lse)
    od = kc.sparse_decode_varlen(s, q, k, v, kv, None)
    torch.cuda.synchronize()
    K = O.topk_count(N, *frac)
    L = s.n_lists
    rows = idx.view(B, L, K).cpu().numpy()
    qn, kn, vn = np64(q), np64(k), np64(v)
    on, ln, odn = np64(o).reshape(B, Hq, d), lse.cpu().numpy(), np64(od).reshape(B, Hq, d)
    name = O.MODES[mode]
    tally = Tally()
    for b, nb in enumerate(lens):
        kb = O.topk_count(nb, *frac)
        assert (rows[b, :, kb:] == -1).all()
        sel = rows[b:b + 1, :, :kb]
        qb, kb_, vb = qn[b:b + 1], kn[b:b + 1, :, :nb], vn[b:b + 1, :, :nb]
        _, pooled = O.anchor_select_decode_mode(qb, kb_, *frac, name)
        for p in range(L):
            tally.add(O.check_index_set(pooled[0, p], kb, sel[0, p]), (b, p))
        ref, lref = O.sparse_decode_mode(qb, kb_, vb, sel, name, None if hm is None else hm.tolist())
        check_out(on[b:b + 1], ref, f"varlen decode row {b}")
        check_lse(ln[b:b + 1], lref, f"varlen lse row {b}")
        G = Hq // Hkv
        for h in range(Hkv):
            dref, _ = O.dense_attention(qb[0, h * G:(h + 1) * G, 0], kb_[0, h], vb[0, h])
            check_out(odn[b, h * G:(h + 1) * G], dref, f"varlen dense row {b}")
    tally.assert_ok()
