"""Failure reporting on the GPU without a fault: a test-only flag makes the
prefill scoring kernel announce a query-tile load that it never issues.  Its
bounded waits give up (a few seconds), the kernel finishes, the call's
workspace error word names the kernel, and the context stays usable."""
import pytest
import torch

import oracle as O
from parity import Tally, gen_inputs, np64, prefill_lists

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_through_the_error_word():
    from sparse_attention_long_anchor_b200 import kascade as kc
    B, Hq, Hkv, d, N, frac = 1, 8, 2, 128, 256, (10, 100)
    q, k, _ = gen_inputs(dict(mode="prefill", B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=9)
    bad = kc.Shape.make(B, Hq, Hkv, d, N, N, frac, flags=kc.FLAG_TEST_DROP_LOAD)
    ws = kc.Workspace(bad)
    kc.select(bad, q, k, ws=ws)                  # launches fine; the device gives up later
    torch.cuda.synchronize()
    assert ws.error(clear=True) == kc.DEVERR_SCORE_POOL
    assert ws.error() == 0                       # cleared
    # the same workspace and context serve a normal call, which is exact
    good = kc.Shape.make(B, Hq, Hkv, d, N, N, frac)
    idx = kc.select(good, q, k, ws=ws)
    torch.cuda.synchronize()
    assert ws.error() == 0
    rows, off = prefill_lists(idx.cpu().numpy(), B, Hkv, N, frac)
    qn, kn = np64(q), np64(k)
    tally = Tally()
    for h in range(Hkv):
        for t in range(len(off) - 1):
            sel = rows[0, h, off[t]:off[t + 1]]
            tally.add(O.check_index_set(O.pooled_prefill_tile(qn, kn, 0, h, t, 32), len(sel), sel), (h, t))
    tally.assert_ok()
