"""The workspace-free decode selection (for callers that can neither pass
device scratch nor allocate) gives the same index sets as kascade_select.

Collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test."""
import ctypes

import pytest
import torch

from parity import gen_inputs

pytestmark = pytest.mark.gpu


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


@pytest.mark.parametrize("B,Hq,Hkv,d,N", [(1, 32, 8, 128, 8192), (2, 8, 2, 64, 3000)])
def test_static_scratch_select_matches_workspace_select(B, Hq, Hkv, d, N):
    kc = _kc()
    q, k, _ = gen_inputs(dict(B=B, Hq=Hq, Hkv=Hkv, d=d, N=N), seed=N + B)
    s = kc.Shape.make(B, Hq, Hkv, d, 1, N, (10, 100))
    assert kc.workspace_bytes(s, kc.OP_SELECT) <= kc.lib.kascade_select_decode_static_max_bytes()
    ref = kc.select(s, q, k, ws=kc.Workspace(s, (kc.OP_SELECT,)))
    first = torch.full_like(ref, -1)
    second = torch.full_like(ref, -1)
    # two calls in a row through the C ABI, sharing the library's array
    for out in (first, second):
        st = kc.lib.kascade_select_decode_static(ctypes.byref(s), q.data_ptr(), k.data_ptr(), out.data_ptr(),
                                                 torch.cuda.current_stream().cuda_stream)
        assert st == kc.OK, kc.status_str(st)
    torch.cuda.synchronize()
    assert torch.equal(first, ref)
    assert torch.equal(second, ref)
    # no bounded wait gave up in either call (the static path's own error word)
    err = ctypes.c_int(-1)
    st = kc.lib.kascade_select_decode_static_error(ctypes.byref(err), 1, torch.cuda.current_stream().cuda_stream)
    assert st == kc.OK and err.value == 0


def test_static_scratch_rejects_oversized_and_prefill_shapes():
    kc = _kc()
    big = kc.Shape.make(8, 32, 8, 128, 1, 65536)   # about 80 MB of scratch
    assert kc.workspace_bytes(big, kc.OP_SELECT) > kc.lib.kascade_select_decode_static_max_bytes()
    st = kc.lib.kascade_select_decode_static(ctypes.byref(big), 256, 256, 256, None)
    assert st == kc.ERR_TOO_LARGE and "scratch" in kc.status_str(st)
    pre = kc.Shape.make(1, 8, 2, 64, 256, 256)
    assert kc.lib.kascade_select_decode_static(ctypes.byref(pre), 256, 256, 256, None) == kc.ERR_UNSUPPORTED
    # shapes kascade_select refuses get the same status here
    for bad in (kc.Shape.make(1, 8, 2, 96, 1, 1024), kc.Shape.make(1, 32, 2, 128, 1, 1024),
                kc.Shape.make(1, 8, 3, 64, 1, 1024), kc.Shape.make(1, 8, 2, 64, 1, 1024, (0, 100))):
        want = kc.lib.kascade_select(ctypes.byref(bad), 256, 256, 256, None, 0, None)
        assert want in (kc.ERR_UNSUPPORTED, kc.ERR_INVALID_ARG)
        assert kc.lib.kascade_select_decode_static(ctypes.byref(bad), 256, 256, 256, None) == want
