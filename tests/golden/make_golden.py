"""Writes the golden fixtures of tests/golden from the fp64 oracle only.

    python tests/golden/make_golden.py

Each fixture stores its input spec (closed-form, see inputs.py), the
oracle's index sets and outputs, and the smallest relative margin between
the k-th and (k+1)-th pooled scores of every selection problem; the script
refuses specs whose margin is below 1e-4, so that index sets compare
bit-exactly."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
sys.path.insert(0, HERE)

import oracle as O  # noqa: E402
from inputs import case  # noqa: E402

SPECS = {
    "decode_tiny": dict(mode="decode", B=1, Hq=4, Hkv=2, d=64, N=40, q_len=1, frac=[25, 100],
                        q_gen=[3, 1, 11], k_gen=[7, 2, 13], v_gen=[5, 3, 9], boost=[0, 9, 17, 33]),
    "prefill_tiny": dict(mode="prefill", B=1, Hq=2, Hkv=1, d=64, N=70, q_len=70, frac=[25, 100],
                         q_gen=[5, 1, 11], k_gen=[7, 4, 13], v_gen=[3, 2, 9], boost=[0, 5, 38, 61]),
}


def margin(pooled, k):
    s = np.sort(np.asarray(pooled))[::-1]
    if k >= len(s):
        return 1.0
    return float((s[k - 1] - s[k]) / s[k - 1])


def build(name, spec):
    q, k, v = case(spec)
    fn, fd = spec["frac"]
    out = {"spec": spec, "source": "fp64 oracle (oracle/kascade_oracle.py)"}
    if spec["mode"] == "decode":
        idx, pooled = O.anchor_select_decode(q, k, fn, fd)
        kk = O.topk_count(spec["N"], fn, fd)
        margins = [margin(pooled[b, h], kk) for b in range(spec["B"]) for h in range(spec["Hkv"])]
        o, lse = O.sparse_decode(q, k, v, idx)
        out.update(idx=np.asarray(idx).tolist(), o=np.round(o, 12).tolist(), lse=np.round(lse, 12).tolist())
    else:
        T = (spec["N"] + 31) // 32
        rows, margins, os_, ls = [], [], [], []
        for t in range(T):
            kt = O.topk_count(min(32 * (t + 1), spec["N"]), fn, fd)
            sel, _ = O.anchor_select_prefill_tile(q, k, 0, 0, t, 32, fn, fd)
            rows.append(np.asarray(sel).tolist())
            margins.append(margin(O.pooled_prefill_tile(q, k, 0, 0, t, 32), kt))
            o, lse = O.sparse_prefill_tile(q, k, v, np.asarray(sel), 0, 0, t, 32)
            os_.append(np.round(o, 12).tolist())
            ls.append(np.round(lse, 12).tolist())
        out.update(tiles=rows, o=os_, lse=ls)
    out["min_margin"] = min(margins)
    assert out["min_margin"] > 1e-4, (name, out["min_margin"])
    return out


if __name__ == "__main__":
    for name, spec in SPECS.items():
        data = build(name, spec)
        with open(os.path.join(HERE, name + ".json"), "w") as f:
            json.dump(data, f)
        print(name, "min margin", data["min_margin"])
