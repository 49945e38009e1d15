"""Small, self-contained cases of the hot-path kernels for profiler captures.

Each case builds seeded synthetic layers with ``synth.make_stack`` and calls
the public binding exactly as a user would (select, then sparse attention),
then times the kernels with CUDA events.  Sizes are chosen so that a capture
of one to three launches holds well under a few GB on the device while the
inputs still exceed the 126 MB L2 where that matters.

    python -m sparse_attention_long_anchor_b200.profile_case decode
    python -m sparse_attention_long_anchor_b200.profile_case prefill --n 8192
    python -m sparse_attention_long_anchor_b200.profile_case decode-batched --n 32768
"""
import argparse

import torch

from . import kascade as kc
from . import synth


def _events():
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def decode_case(reps: int = 20) -> None:
    """Llama-shaped decode (B=1, Hq=32, Hkv=8, d=128, N=32768): one anchor
    select on layer 0 and sparse decode of reuse layers 1..3."""
    cfg = synth.CONFIGS["decode_llama8b_n32k"]
    plan, L = synth.make_stack(cfg, device="cuda", layers=[0, 1, 2, 3])
    s = kc.Shape.make(cfg.batch, cfg.hq, cfg.hkv, cfg.d, 1, cfg.n_ctx)
    ws = kc.Workspace(s)
    idx = kc.select(s, L[0][0], L[0][1], ws=ws)
    hm = torch.tensor(plan[1][2], dtype=torch.int32, device="cuda")
    for _ in range(3):
        for l in (1, 2, 3):
            kc.sparse_decode(s, L[l][0], L[l][1], L[l][2], idx, hm, ws=ws)
        kc.select(s, L[0][0], L[0][1], idx, ws=ws)
    torch.cuda.synchronize()
    e0, e1 = _events()
    e0.record()
    for _ in range(reps):
        for l in (1, 2, 3):
            kc.sparse_decode(s, L[l][0], L[l][1], L[l][2], idx, hm, ws=ws)
    e1.record()
    torch.cuda.synchronize()
    print(f"sparse decode eager us/launch {e0.elapsed_time(e1) * 1e3 / (3 * reps):.2f}")
    e0.record()
    for _ in range(reps):
        kc.select(s, L[0][0], L[0][1], idx, ws=ws)
    e1.record()
    torch.cuda.synchronize()
    print(f"select eager us/launch {e0.elapsed_time(e1) * 1e3 / reps:.2f}")
    err = ws.error()
    if err:
        raise RuntimeError(f"device error word {err}")


def decode_batched_case(n: int = 32768, reps: int = 10) -> None:
    """Batched Llama-shaped decode (B=8, Hq=32, Hkv=8, d=128) at context n:
    one anchor select on layer 0, sparse decode of reuse layers 1 and 2
    alternating (at n = 32768 they gather 2 x 108 MB, beyond L2; 3.2 GB of
    K/V on the device)."""
    cfg = synth.CONFIGS["decode_llama8b_b8_n64k"].with_(n_ctx=n, n_layers=3)
    plan, L = synth.make_stack(cfg, device="cuda", layers=[0, 1, 2])
    s = kc.Shape.make(cfg.batch, cfg.hq, cfg.hkv, cfg.d, 1, cfg.n_ctx)
    ws = kc.Workspace(s)
    idx = kc.select(s, L[0][0], L[0][1], ws=ws)
    hms = {l: torch.tensor(plan[l][2], dtype=torch.int32, device="cuda") for l in (1, 2)}
    for _ in range(2):
        for l in (1, 2):
            kc.sparse_decode(s, L[l][0], L[l][1], L[l][2], idx, hms[l], ws=ws)
        kc.select(s, L[0][0], L[0][1], idx, ws=ws)
    torch.cuda.synchronize()
    e0, e1 = _events()
    e0.record()
    for _ in range(reps):
        for l in (1, 2):
            kc.sparse_decode(s, L[l][0], L[l][1], L[l][2], idx, hms[l], ws=ws)
    e1.record()
    torch.cuda.synchronize()
    print(f"batched sparse decode eager us/launch {e0.elapsed_time(e1) * 1e3 / (2 * reps):.2f}")
    e0.record()
    for _ in range(reps):
        kc.select(s, L[0][0], L[0][1], idx, ws=ws)
    e1.record()
    torch.cuda.synchronize()
    print(f"batched select eager us/launch {e0.elapsed_time(e1) * 1e3 / reps:.2f}")
    err = ws.error()
    if err:
        raise RuntimeError(f"device error word {err}")


def prefill_case(n: int = 8192, reps: int = 2) -> None:
    """Qwen-shaped causal prefill (Hq=32, Hkv=8, d=128) at context n: anchor
    select on layer 0, sparse prefill of reuse layer 1."""
    cfg = synth.CONFIGS["prefill_qwen8b_n32k"].with_(n_ctx=n, n_layers=2)
    plan, L = synth.make_stack(cfg, device="cuda", layers=[0, 1])
    s = kc.Shape.make(cfg.batch, cfg.hq, cfg.hkv, cfg.d, n, n)
    ws = kc.Workspace(s)
    hm = torch.tensor(plan[1][2], dtype=torch.int32, device="cuda")
    q, k, _ = L[0]
    idx = kc.select(s, q, k, ws=ws)
    for _ in range(reps):
        kc.select(s, q, k, idx, ws=ws)
        kc.sparse_prefill(s, L[1][0], L[1][1], L[1][2], idx, hm, ws=ws)
    torch.cuda.synchronize()
    e0, e1 = _events()
    e0.record()
    kc.select(s, q, k, idx, ws=ws)
    e1.record()
    torch.cuda.synchronize()
    print(f"select ms {e0.elapsed_time(e1):.3f}")
    e0.record()
    kc.sparse_prefill(s, L[1][0], L[1][1], L[1][2], idx, hm, ws=ws)
    e1.record()
    torch.cuda.synchronize()
    print(f"sparse prefill ms {e0.elapsed_time(e1):.3f}")
    err = ws.error()
    if err:
        raise RuntimeError(f"device error word {err}")


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["decode", "prefill", "decode-batched"])
    ap.add_argument("--n", type=int, default=None,
                    help="context length (prefill: default 8192; decode-batched: default 32768)")
    a = ap.parse_args()
    if a.case == "decode":
        decode_case()
    elif a.case == "decode-batched":
        decode_batched_case(a.n or 32768)
    else:
        prefill_case(a.n or 8192)
    print("ok")


if __name__ == "__main__":
    main()
