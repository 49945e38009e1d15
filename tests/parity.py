"""Helpers for the GPU-vs-oracle parity tests.

Tolerances for bf16 outputs: max-abs 2e-2 and mean-abs 2e-3 against the fp64
oracle evaluated on the GPU's own index set.  Index sets are judged with the
oracle's acceptance rule (exact, or a near tie within 1e-6 relative)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 2e-3


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_out(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def check_lse(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    fin = np.isfinite(want)
    assert np.array_equal(fin, np.isfinite(got)), f"{what}: -inf pattern differs"
    if fin.any():
        err = np.abs(got[fin] - want[fin]).max()
        assert err <= LSE_ABS, f"{what}: lse err {err:.3e}"
    assert np.all(got[~fin] == -np.inf)


class Tally:
    def __init__(self):
        self.counts = {"exact": 0, "near_tie": 0, "fail": 0}
        self.fails = []

    def add(self, verdict, info=None):
        self.counts[verdict] += 1
        if verdict == "fail":
            self.fails.append(info)

    def assert_ok(self):
        assert self.counts["fail"] == 0, f"index sets failed: {self.fails[:5]} counts={self.counts}"


def decode_idx_check(qn, kn, idx_gpu, frac, tally=None):
    """Judge every (b, h) decode index set; returns the oracle's sets."""
    tally = tally or Tally()
    bsz, hkv = kn.shape[0], kn.shape[1]
    kk = O.topk_count(kn.shape[2], *frac)
    idx_o, pooled = O.anchor_select_decode(qn, kn, *frac)
    for b in range(bsz):
        for h in range(hkv):
            v = O.check_index_set(pooled[b, h], kk, idx_gpu[b, h])
            tally.add(v, (b, h))
    return idx_o, tally


def prefill_lists(idx_flat: np.ndarray, bsz, hkv, n_ctx, frac):
    """Split the flat prefill index buffer into per-(b, h) rows and tiles."""
    off = O.index_offsets(n_ctx, 32, *frac)
    rows = idx_flat.reshape(bsz, hkv, int(off[-1]))
    return rows, off


def gen_inputs(shape_kw, seed=0, device="cuda", zero_q=False, band=None, n_salient=64):
    """Seeded synthetic Q, K, V of one layer (the workloads' recipe)."""
    from sparse_attention_long_anchor_b200 import synth
    if band is None:
        band = shape_kw.get("mode", "decode") == "prefill"
    cfg = synth.StackConfig("t", shape_kw.get("mode", "decode"), shape_kw["B"], shape_kw["Hq"],
                            shape_kw["Hkv"], shape_kw["d"], shape_kw["N"], 1, (0,), band=band,
                            n_salient=n_salient, seed=seed)
    sal = synth.salient_sets(cfg)[0]
    q, k, v = synth.make_layer(cfg, 0, sal, device)
    if zero_q:
        q = torch.zeros_like(q)
    return q, k, v
