"""The C ABI library loads, exports every symbol that include/kascade.h
declares, and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "kascade.h")).read()
    return re.findall(r"KASCADE_API\s+[\w\s\*]+?\b(kascade_\w+)\s*\(", txt)


def test_library_exports_every_declared_symbol():
    from sparse_attention_long_anchor_b200 import kascade as kc
    names = _declared()
    assert len(names) >= 10
    assert set(names) == set(kc.EXPORTS)
    for n in names:
        assert hasattr(kc.lib, n), n


def _kc():
    from sparse_attention_long_anchor_b200 import kascade as kc
    return kc


@pytest.mark.parametrize("n_ctx", [1, 31, 32, 33, 100, 2048, 32768, 131072])
@pytest.mark.parametrize("frac", [(10, 100), (5, 100), (20, 100), (1, 1), (1, 3)])
def test_index_layout_matches_oracle(n_ctx, frac):
    kc = _kc()
    s = kc.Shape.make(2, 8, 2, 128, n_ctx, n_ctx, frac)
    off = kc.index_offsets(s)
    want = O.index_offsets(n_ctx, 32, *frac)
    assert off.tolist() == want.tolist()
    assert kc.index_count(s) == 2 * 2 * int(want[-1])
    d = kc.Shape.make(2, 8, 2, 128, 1, n_ctx, frac)
    assert kc.index_count(d) == 2 * 2 * O.topk_count(n_ctx, *frac)
    assert kc.index_offsets(d).tolist() == [0, O.topk_count(n_ctx, *frac)]


def test_workspace_sizes_positive():
    kc = _kc()
    s = kc.Shape.make(1, 32, 8, 128, 1, 32768)
    assert kc.workspace_bytes(s, kc.OP_SELECT) > 256
    for op in (kc.OP_SPARSE_DECODE, kc.OP_SPARSE_PREFILL, kc.OP_DENSE):
        assert kc.workspace_bytes(s, op) == 256
    p = kc.Shape.make(1, 32, 8, 128, 32768, 32768)
    assert kc.workspace_bytes(p, kc.OP_SELECT) > 0


@pytest.mark.parametrize("bad,status", [
    (dict(head_dim=96), 2), (dict(head_dim=0), 2), (dict(num_q_heads=12, num_kv_heads=8), 1),
    (dict(num_q_heads=64, num_kv_heads=4), 2), (dict(topk_num=0), 1), (dict(topk_num=11, topk_den=10), 1),
    (dict(tile=16, q_len=64, kv_len=64), 2), (dict(q_len=7), 2), (dict(batch=0), 1), (dict(kv_len=0), 1),
    (dict(select_mode=3), 1), (dict(select_mode=-1), 1), (dict(dtype=3), 2),
    (dict(select_mode=2, num_q_heads=128, num_kv_heads=64), 2),
])
def test_bad_shapes_are_rejected(bad, status):
    kc = _kc()
    s = kc.Shape.make(1, 8, 2, 64, 1, 256)
    for key, val in bad.items():
        setattr(s, key, val)
    assert kc.workspace_bytes(s, kc.OP_SELECT) == 0
    assert kc.lib.kascade_select(ctypes.byref(s), 256, 256, 256, 256, 1 << 30, None) == status
    assert kc.lib.kascade_index_count(ctypes.byref(s)) == -1


def test_null_and_misaligned_pointers_and_small_workspace():
    kc = _kc()
    s = kc.Shape.make(1, 8, 2, 64, 1, 256)
    L = kc.lib
    sb = ctypes.byref(s)
    need = kc.workspace_bytes(s, kc.OP_SELECT)
    assert L.kascade_select(sb, None, 256, 256, 256, need, None) == kc.ERR_INVALID_ARG
    assert L.kascade_select(sb, 256, 256, None, 256, need, None) == kc.ERR_INVALID_ARG
    assert L.kascade_select(sb, 258, 256, 256, 256, need, None) == kc.ERR_UNSUPPORTED
    assert L.kascade_select(sb, 256, 256, 256, 256, need - 1, None) == kc.ERR_WORKSPACE
    assert L.kascade_select(sb, 256, 256, 256, None, need, None) == kc.ERR_WORKSPACE
    assert L.kascade_select(sb, 256, 256, 256, 258, need, None) == kc.ERR_WORKSPACE
    nd = kc.workspace_bytes(s, kc.OP_SPARSE_DECODE)
    assert nd == 256   # only the error-word header: attention partials stay on chip
    assert L.kascade_sparse_decode(sb, 256, 256, 256, None, None, 256, None, None, 0, None) == kc.ERR_INVALID_ARG
    assert L.kascade_sparse_decode(sb, 256, 256, None, 256, None, 256, None, None, 0, None) == kc.ERR_INVALID_ARG
    assert L.kascade_sparse_decode(sb, None, 256, 256, 256, None, 256, None, None, 0, None) == kc.ERR_INVALID_ARG
    assert L.kascade_sparse_decode(sb, 256, 256, 256, 258, None, 256, None, None, 0, None) == kc.ERR_UNSUPPORTED
    assert L.kascade_sparse_decode(sb, 256, 264, 256, 256, None, 256, None, None, 0, None) == kc.ERR_UNSUPPORTED
    # prefill entry points refuse decode shapes and vice versa
    assert L.kascade_sparse_prefill(sb, 256, 256, 256, 256, None, 256, None, None, 0, None) == kc.ERR_UNSUPPORTED
    p = kc.Shape.make(1, 8, 2, 64, 256, 256)
    assert L.kascade_sparse_decode(ctypes.byref(p), 256, 256, 256, 256, None, 256, None, 256, nd, None) \
        == kc.ERR_UNSUPPORTED
    assert L.kascade_workspace_init(None, 16, None) == kc.ERR_WORKSPACE
    assert L.kascade_index_offsets(sb, None) == kc.ERR_INVALID_ARG
    out = ctypes.c_int(0)
    assert L.kascade_workspace_error(None, ctypes.byref(out), 0, None) == kc.ERR_INVALID_ARG
    assert L.kascade_workspace_error(256, None, 0, None) == kc.ERR_INVALID_ARG


def test_status_strings():
    kc = _kc()
    for st in range(5):
        assert isinstance(kc.status_str(st), str) and kc.status_str(st)
    assert kc.status_str(99) == "unknown status"


@pytest.mark.parametrize("mode,lists", [(0, 2), (1, 8), (2, 1)])
def test_index_layout_per_selection_mode(mode, lists):
    """L lists per batch row: Hkv (GQA), Hq (per query head), 1 (all heads)."""
    kc = _kc()
    d = kc.Shape.make(3, 8, 2, 64, 1, 1000, mode=mode)
    assert d.n_lists == lists
    assert kc.index_count(d) == 3 * lists * O.topk_count(1000, 10, 100)
    p = kc.Shape.make(3, 8, 2, 64, 1000, 1000, mode=mode)
    assert kc.index_count(p) == 3 * lists * int(O.index_offsets(1000, 32, 10, 100)[-1])
    for dt in (0, 1, 2):
        for sh in (d, p):
            sh.dtype = dt
            assert kc.workspace_bytes(sh, kc.OP_SELECT) > 0


def test_index_check_flag_workspace_and_launches():
    """KASCADE_FLAG_CHECK_INDICES: the attention and refine workspaces grow by
    the checked copies (lists, head_map, kv_lens), the attention calls count
    one more launch, and a call without a workspace large enough is refused
    on the host."""
    kc = _kc()
    for q_len, n in ((1, 32768), (4096, 4096), (64, 4096)):
        s = kc.Shape.make(2, 32, 8, 128, q_len, n)
        c = s.with_flags(kc.FLAG_CHECK_INDICES)
        entries = kc.index_count(s)
        for op in (kc.OP_SPARSE_DECODE, kc.OP_SPARSE_PREFILL):
            assert kc.workspace_bytes(c, op) >= 256 + 4 * entries + 4 * 32 + 4 * 2
            assert kc.workspace_bytes(c, op) % 256 == 0
            assert kc.launch_count(c, op) == 2 and kc.launch_count(s, op) == 1
        assert kc.workspace_bytes(c, kc.OP_DENSE) == 256 and kc.launch_count(c, kc.OP_DENSE) == 1
        if q_len == 1:
            assert kc.workspace_bytes(c, kc.OP_REFINE) >= kc.workspace_bytes(s, kc.OP_REFINE) + 4 * 2 * 8 * n
    s = kc.Shape.make(1, 8, 2, 64, 1, 256).with_flags(kc.FLAG_CHECK_INDICES)
    need = kc.workspace_bytes(s, kc.OP_SPARSE_DECODE)
    L = kc.lib
    args = (ctypes.byref(s), 256, 256, 256, 256, None, 256, None)
    assert L.kascade_sparse_decode(*args, None, 0, None) == kc.ERR_WORKSPACE
    assert L.kascade_sparse_decode(*args, 256, need - 1, None) == kc.ERR_WORKSPACE
    assert L.kascade_sparse_decode(*args, 258, need, None) == kc.ERR_WORKSPACE
    p = kc.Shape.make(1, 8, 2, 64, 256, 256).with_flags(kc.FLAG_CHECK_INDICES)
    assert L.kascade_sparse_prefill(ctypes.byref(p), 256, 256, 256, 256, None, 256, None, None, 0, None) \
        == kc.ERR_WORKSPACE
