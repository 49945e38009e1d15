"""Stored fixtures (tests/golden, written by make_golden.py from the fp64
oracle on closed-form inputs with clear top-k margins).

CPU: the oracle still reproduces them (a regression pin on the oracle).
GPU: the CUDA path matches the stored index sets bit for bit and the stored
outputs within the bf16 tolerances."""
import json
import os
import sys

import numpy as np
import pytest
import torch

import oracle as O
from parity import check_lse, check_out

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
sys.path.insert(0, HERE)
from inputs import case  # noqa: E402

NAMES = ["decode_tiny", "prefill_tiny"]


def load(name):
    with open(os.path.join(HERE, name + ".json")) as f:
        return json.load(f)


@pytest.mark.parametrize("name", NAMES)
def test_oracle_reproduces_golden(name):
    g = load(name)
    spec = g["spec"]
    q, k, v = case(spec)
    fn, fd = spec["frac"]
    if spec["mode"] == "decode":
        idx, _ = O.anchor_select_decode(q, k, fn, fd)
        assert np.array_equal(np.asarray(idx), np.asarray(g["idx"]))
        o, lse = O.sparse_decode(q, k, v, idx)
        assert np.abs(o - np.asarray(g["o"])).max() < 1e-9
        assert np.abs(lse - np.asarray(g["lse"])).max() < 1e-9
    else:
        for t, want in enumerate(g["tiles"]):
            sel, _ = O.anchor_select_prefill_tile(q, k, 0, 0, t, 32, fn, fd)
            assert np.array_equal(np.asarray(sel), np.asarray(want)), t
            o, lse = O.sparse_prefill_tile(q, k, v, np.asarray(sel), 0, 0, t, 32)
            assert np.abs(o - np.asarray(g["o"][t])).max() < 1e-9


def _dev(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).cuda().contiguous()


@pytest.mark.gpu
@pytest.mark.parametrize("name", NAMES)
def test_cuda_matches_golden(name):
    from sparse_attention_long_anchor_b200 import kascade as kc
    g = load(name)
    spec = g["spec"]
    q, k, v = case(spec)
    qd, kd, vd = _dev(q), _dev(k), _dev(v)
    frac = tuple(spec["frac"])
    B, Hq, Hkv, d, N, L = spec["B"], spec["Hq"], spec["Hkv"], spec["d"], spec["N"], spec["q_len"]
    s = kc.Shape.make(B, Hq, Hkv, d, L, N, frac)
    ws = kc.Workspace(s)
    idx = kc.select(s, qd, kd, ws=ws)
    lse = torch.empty(B, Hq, L, device="cuda")
    if spec["mode"] == "decode":
        o = kc.sparse_decode(s, qd, kd, vd, idx, None, lse=lse, ws=ws)
        torch.cuda.synchronize()
        got = idx.view(B, Hkv, -1).cpu().numpy()
        assert np.array_equal(got, np.asarray(g["idx"]))
        check_out(o.float().cpu().numpy().reshape(B, Hq, d), np.asarray(g["o"]), name)
        check_lse(lse.cpu().numpy().reshape(B, Hq), np.asarray(g["lse"]), name)
    else:
        o = kc.sparse_prefill(s, qd, kd, vd, idx, None, lse=lse, ws=ws)
        torch.cuda.synchronize()
        off = O.index_offsets(N, 32, *frac)
        flat = idx.cpu().numpy()
        on = o.float().cpu().numpy()
        for t, want in enumerate(g["tiles"]):
            assert np.array_equal(flat[off[t]:off[t + 1]], np.asarray(want)), t
            i0, i1 = 32 * t, min(32 * t + 32, N)
            check_out(on[0, :, i0:i1], np.asarray(g["o"][t]), f"{name} tile {t}")
    assert ws.error() == 0
