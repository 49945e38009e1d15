"""Benchmark of the Kascade hot path on B200.

One step = one decode step of the 32-layer Llama-3.1-8B-shaped stack
(B=1, Hq=32, Hkv=8, d=128, N=32768, Top-k 10 %, anchors {0, 8, 16, 24}) and
one causal prefill of the 36-layer Qwen3-8B-shaped stack (N=32768, tile 32,
anchors {0, 9, 18, 27}), each captured as a CUDA graph.  The headline value is
sparse decode microseconds per layer-step; the prefill figure (ms per layer)
rides along in the same JSON line.

After the timed steps the other workloads are timed the same way, each as a
CUDA graph of its whole stack, and reported under ``configs``: the 2-layer
2K decode, the batched decode (8 sequences of 64K, the full 32-layer stack),
and the 128K prefill (1 anchor + 7 reuse layers) at Top-k 5, 10 and 20 %.
The library's own dense attention is timed on the 32K decode and prefill
layers as the on-box dense denominator.

Inputs are seeded synthetic tensors generated on the device; every layer has
its own KV (4.3 GB decode, 14.5 GB prefill per GPU), far larger than the
126 MB L2, so no L2 flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kascade|reference]

Under torchrun every rank runs its own replica of the workload (independent
batches, no data-path collective: weak scaling); times are the max over
ranks.  ``--impl reference`` times the fp64 CPU oracle on the host cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse decode µs/layer-step & prefill ms/layer at 32K-128K ctx; % HBM/TC roofline"
DECODE_CFG = "decode_llama8b_n32k"
PREFILL_CFG = "prefill_qwen8b_n32k"
SMALL_DECODE_CFG = "decode_b1_h8_n2k"
BATCHED_DECODE_CFG = "decode_llama8b_b8_n64k"
LONG_PREFILL_CFG = "prefill_n128k"
LONG_PREFILL_FRACS = ((5, 100), (10, 100), (20, 100))


# ----------------------------------------------------------------------------- helpers


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def strip_comments(src: str) -> str:
    """C/C++/CUDA source without its comments and blank-line or indentation
    differences: string and character literals are kept as they are, every
    comment is dropped, and each remaining line is stripped of surrounding
    whitespace (empty lines dropped)."""
    out, i, n = [], 0, len(src)
    while i < n:
        ch = src[i]
        if ch in "\"'":
            j = i + 1
            while j < n and src[j] != ch:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(ch)
            i += 1
    lines = (ln.strip() for ln in "".join(out).splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_source_hash(name: str) -> str:
    """Hash of a kernel source's code (comments and layout ignored), which
    keys the stored ncu counters to the code they were taken on."""
    import hashlib
    path = os.path.join(ROOT, "sparse_attention_long_anchor_b200", "csrc", name)
    with open(path, encoding="utf-8") as f:
        return hashlib.sha256(strip_comments(f.read()).encode()).hexdigest()[:16]


def profiled_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from one ncu capture, kept in
    profiles/traffic.json with the hash of the kernel's source; None when the
    source changed after the capture (the counters no longer describe it)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            entry = json.load(f)[kernel]
        if entry["source_sha"] != kernel_source_hash(entry["source"]):
            return None
        return float(entry["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError, TypeError):
        return None


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 6:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[2:6]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local) if torch.cuda.is_available() else None
        dist.init_process_group("nccl" if torch.cuda.is_available() else "gloo",
                                timeout=datetime.timedelta(seconds=600))
    return rank, world, local


def dist_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def spread(xs):
    """median, p10 and p90 of a list of timings."""
    s = sorted(xs)
    if not s:
        return {"median": None, "p10": None, "p90": None, "n": 0}

    def q(f):
        return s[min(len(s) - 1, max(0, int(round(f * (len(s) - 1)))))]
    return {"median": statistics.median(s), "p10": q(0.1), "p90": q(0.9), "n": len(s)}


# ----------------------------------------------------------------------------- oracle timing


def host_cores():
    """Host cores: what the process may run on, and the CPU model."""
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count() or 1
    model = platform.processor() or ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": usable, "cpu_count": os.cpu_count(), "model": model}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] + [1])
    except Exception:
        return os.cpu_count() or 1


def host_copy_layer(q, k, v):
    import numpy as np
    return tuple(t.float().cpu().numpy().astype(np.float64) for t in (q, k, v))


def oracle_decode_sample(cfg, layers_np, plan):
    """The oracle on one anchor layer and one reuse layer of the decode
    stack.  Returns (weighted µs per layer-step of the stack, seconds the
    sample took, detail)."""
    import oracle as O
    frac = (cfg.frac_num, cfg.frac_den)
    (q0, k0, v0), (q1, k1, v1) = layers_np
    t0 = time.perf_counter()
    idx, _ = O.anchor_select_decode(q0, k0, *frac)
    O.sparse_decode(q0, k0, v0, idx)
    t1 = time.perf_counter()
    O.sparse_decode(q1, k1, v1, idx, plan[1][2])
    t2 = time.perf_counter()
    anchor_s, reuse_s = t1 - t0, t2 - t1
    n_anchor = sum(1 for p in plan if p[0])
    n_reuse = len(plan) - n_anchor
    per_layer = (n_anchor * anchor_s + n_reuse * reuse_s) / len(plan)
    return per_layer * 1e6, t2 - t0, {"anchor_layer_s": anchor_s, "reuse_layer_s": reuse_s}


def oracle_prefill_sample(cfg, layers_np, plan, n_random=12, seed=0):
    """The oracle on a seeded sample of one anchor layer's tile problems
    (tiles {0, 1, 2, T-1} plus `n_random` random tiles, kv head 0: pooling,
    Top-k and the anchor's own sparse attention) and the same tiles of the
    following reuse layer.  Per-tile cost grows with the tile's candidate
    count e_t (anchor) and list length k_t (reuse); the full-layer times are
    extrapolated from the sample by those counts and labelled so."""
    import numpy as np

    import oracle as O
    frac = (cfg.frac_num, cfg.frac_den)
    (q0, k0, v0), (q1, k1, v1) = layers_np
    T = -(-cfg.n_ctx // cfg.tile)
    rng = np.random.default_rng(seed)
    tiles = sorted(set([0, 1, 2, T - 1] + rng.choice(np.arange(3, T - 1), n_random, replace=False).tolist()))
    e = O.tile_ends(cfg.n_ctx, cfg.tile)
    kt = O.tile_topk_counts(cfg.n_ctx, cfg.tile, *frac)
    hm1 = plan[1][2]
    a_s, r_s = 0.0, 0.0
    for t in tiles:
        t0 = time.perf_counter()
        sel, _ = O.anchor_select_prefill_tile(q0, k0, 0, 0, t, cfg.tile, *frac)
        O.sparse_prefill_tile(q0, k0, v0, sel, 0, 0, t, cfg.tile)
        t1 = time.perf_counter()
        # the reuse layer's kv head h with head_map[h] == 0 reads this list
        h = hm1.index(0) if 0 in hm1 else 0
        O.sparse_prefill_tile(q1, k1, v1, sel, 0, h, t, cfg.tile)
        t2 = time.perf_counter()
        a_s += t1 - t0
        r_s += t2 - t1
    a_per_key = a_s / sum(e[t] for t in tiles)
    r_per_key = r_s / sum(kt[t] for t in tiles)
    anchor_ms = a_per_key * sum(e) * cfg.hkv * cfg.batch * 1e3
    reuse_ms = r_per_key * sum(kt) * cfg.hkv * cfg.batch * 1e3
    n_anchor = len(cfg.anchors)
    per_layer = (n_anchor * anchor_ms + (cfg.n_layers - n_anchor) * reuse_ms) / cfg.n_layers
    return {"sample": f"kv head 0, tiles {tiles} of anchor layer 0 (pool, Top-k, own attention) and reuse layer 1",
            "tile_problems": len(tiles), "sample_s": a_s + r_s,
            "anchor_s_per_tile_problem": a_s / len(tiles), "reuse_s_per_tile_problem": r_s / len(tiles),
            "extrapolated_anchor_layer_ms": anchor_ms, "extrapolated_reuse_layer_ms": reuse_ms,
            "extrapolated_ms_per_layer": per_layer,
            "label": "extrapolated from the sample by candidate and list counts"}


def cpu_baseline_block(dcfg, dlayers, dplan, pcfg=None, players=None, pplan=None):
    """The oracle as it stands on the host cores: decode sample on all
    cores and on one thread; prefill sample (all cores) when given."""
    L = [host_copy_layer(*dlayers[0]), host_copy_layer(*dlayers[1])]
    v_all, s_all, detail = oracle_decode_sample(dcfg, L, dplan)
    v_one = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            v_one, _, _ = oracle_decode_sample(dcfg, L, dplan)
    except Exception:
        pass
    hc = host_cores()
    out = {"value": v_all, "unit": "us/layer-step", "cores": blas_threads(), "cores_nproc": hc["nproc"],
           "cpu_model": hc["model"], "kind": "oracle", "value_1thread": v_one,
           "sample": "oracle (fp64 numpy) on anchor layer 0 and reuse layer 1 of the 32K decode stack, weighted "
                     "4 anchor : 28 reuse layers; " + json.dumps({k: round(x, 4) for k, x in detail.items()})}
    if pcfg is not None:
        P = [host_copy_layer(*players[0]), host_copy_layer(*players[1])]
        out["prefill"] = oracle_prefill_sample(pcfg, P, pplan)
    return out


# ----------------------------------------------------------------------------- reference arm


def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores: every step runs the
    oracle on anchor layer 0 and reuse layer 1 of the 32K decode stack (a
    bounded sample of the step).  ms_per_step is the time those two layers
    took; value is the stack's µs per layer-step with the two layers weighted
    4 anchors : 28 reuse layers."""
    if rank != 0:
        return
    import numpy as np
    from sparse_attention_long_anchor_b200 import synth
    cfg = synth.CONFIGS[DECODE_CFG]
    plan, layers = synth.make_stack(cfg, device="cpu", layers=[0, 1])
    L = [host_copy_layer(*layers[0]), host_copy_layer(*layers[1])]
    vals, secs = [], []
    for step in range(args.warmup + args.steps):
        v, s, _ = oracle_decode_sample(cfg, L, plan)
        if step >= args.warmup:
            vals.append(v)
            secs.append(s)
    value = float(np.mean(vals))
    hc = host_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "us/layer-step", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": float(np.mean(secs)) * 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": DECODE_CFG, "global_batch": cfg.batch, "seq_len": cfg.n_ctx, "layers": cfg.n_layers,
                   "parallelism": f"replicas{world}",
                   "step": "oracle on anchor layer 0 + reuse layer 1 (ms_per_step is their measured time)"},
        "cpu_baseline": {"value": value, "unit": "us/layer-step", "cores": blas_threads(),
                         "cores_nproc": hc["nproc"], "cpu_model": hc["model"], "kind": "oracle",
                         "sample": "per step: oracle on anchor layer 0 and reuse layer 1 of the stack, weighted "
                                   "4 anchor : 28 reuse layers"},
        "e2e": {"value": value, "unit": "us/layer-step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- kascade arm


def build_stack(kc, synth, torch, dev, name, frac=None, layers=None):
    """A stack's tensors, shape (with programmatic dependent launch), one
    workspace, index buffers per anchor, head maps and outputs."""
    cfg = synth.CONFIGS[name]
    if frac is not None:
        cfg = cfg.with_(frac_num=frac[0], frac_den=frac[1])
    plan, ls = synth.make_stack(cfg, device=dev, layers=layers)
    fr = (cfg.frac_num, cfg.frac_den)
    shape = kc.Shape.make(cfg.batch, cfg.hq, cfg.hkv, cfg.d, cfg.q_len, cfg.n_ctx, fr, flags=kc.FLAG_PDL)
    ws = kc.Workspace(shape, device=dev)
    idx = {a: torch.empty(kc.index_count(shape), dtype=torch.int32, device=dev) for a in cfg.anchors}
    hms = {l: torch.tensor(p[2], dtype=torch.int32, device=dev) for l, p in enumerate(plan) if not p[0]}
    outs = {l: torch.empty_like(ls[l][0]) for l in ls}
    return {"cfg": cfg, "plan": plan, "layers": ls, "shape": shape, "ws": ws, "idx": idx, "hms": hms, "outs": outs,
            "stable": shape.with_flags(kc.FLAG_PDL | kc.FLAG_INPUTS_STABLE)}


def run_layer(kc, st, l, which="all"):
    """One layer of a stack.  Kernels use programmatic dependent launch; a
    decode reuse layer reads an index set written at least two launches
    earlier and a KV cache that no kernel of the step writes, so its gathers
    may start early."""
    cfg, plan = st["cfg"], st["plan"]
    is_anchor, anchor, _ = plan[l]
    q, k, v = st["layers"][l]
    decode = cfg.mode == "decode"
    attn = kc.sparse_decode if decode else kc.sparse_prefill
    if is_anchor:
        if which in ("all", "select"):
            kc.select(st["shape"], q, k, st["idx"][l], ws=st["ws"])
        if which in ("all", "attn"):
            attn(st["shape"], q, k, v, st["idx"][l], None, o=st["outs"][l], ws=st["ws"])
    elif which in ("all", "attn"):
        attn(st["stable"] if decode else st["shape"], q, k, v, st["idx"][anchor], st["hms"][l], o=st["outs"][l],
             ws=st["ws"])


def capture(torch, fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()          # warm the launch configuration outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def time_graph(torch, g, reps):
    """Per-replay times (ms) of a graph, CUDA events on the launching stream."""
    g.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for e0, e1 in ev:
        e0.record()
        g.replay()
        e1.record()
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in ev]


def mean(xs):
    return sum(xs) / len(xs)


def decode_bytes(cfg):
    """Algorithmic bytes of one decode layer: (reuse layer, anchor layer's K
    stream): reuse = B Hkv (2 k d 2 + 4 k); the anchor adds its full K."""
    kk = math.ceil(cfg.frac_num * cfg.n_ctx / cfg.frac_den)
    reuse = cfg.batch * cfg.hkv * (2 * kk * cfg.d * 2 + 4 * kk)
    anchor_score = cfg.batch * cfg.hkv * cfg.n_ctx * cfg.d * 2
    return kk, reuse, anchor_score


def prefill_flops(cfg):
    """Executed flops of the two-pass exact scoring of one anchor layer,
    gathered bytes and flops of one sparse prefill layer."""
    T = math.ceil(cfg.n_ctx / cfg.tile)
    e = [min(cfg.tile * (t + 1), cfg.n_ctx) for t in range(T)]
    kt = [math.ceil(cfg.frac_num * x / cfg.frac_den) for x in e]
    one_pass = sum(2 * cfg.hq * cfg.d * cfg.tile * x for x in e)
    gather = sum(cfg.batch * cfg.hkv * 2 * k * cfg.d * 2 for k in kt)
    sparse_flops = sum(cfg.batch * cfg.hq * 4 * cfg.tile * k * cfg.d for k in kt)
    return 2 * one_pass * cfg.batch, one_pass * cfg.batch, gather, sparse_flops


def decode_components(kc, torch, st, reps, pk):
    """Sparse decode per launch and anchor select per anchor of a decode
    stack, each as a graph of only those launches, plus the layer-step
    roofline over the whole stack time."""
    cfg = st["cfg"]
    n = cfg.n_layers
    g_attn = capture(torch, lambda: [run_layer(kc, st, l, "attn") for l in range(n)])
    g_sel = capture(torch, lambda: [run_layer(kc, st, l, "select") for l in range(n)])
    attn = time_graph(torch, g_attn, reps)
    sel = time_graph(torch, g_sel, reps)
    del g_attn, g_sel
    kk, reuse_bytes, score_bytes = decode_bytes(cfg)
    n_anchor = len(cfg.anchors)
    attn_us = mean(attn) * 1e3 / n
    sel_us = mean(sel) * 1e3 / n_anchor
    gbs = reuse_bytes / (attn_us * 1e-6) / 1e9
    return {"sparse_decode_us_per_launch": attn_us, "sparse_decode_algorithmic_bytes": reuse_bytes,
            "sparse_decode_GBps": gbs, "sparse_decode_frac_of_hbm": gbs / pk["hbm_gbs"],
            "anchor_select_us": sel_us, "anchor_select_GBps_on_K": score_bytes / (sel_us * 1e-6) / 1e9,
            "anchor_select_frac_of_hbm_on_K": score_bytes / (sel_us * 1e-6) / 1e9 / pk["hbm_gbs"]}


def step_bytes_decode(cfg):
    """Algorithmic bytes of a whole decode step: reuse layers move K_S + V_S
    + idx, anchors their full K plus V_S + idx."""
    kk, reuse, score = decode_bytes(cfg)
    n_anchor = len(cfg.anchors)
    return (cfg.n_layers - n_anchor) * reuse + n_anchor * (score + cfg.batch * cfg.hkv * (kk * cfg.d * 2 + 4 * kk))


def time_decode_stack(kc, torch, st, reps, pk, with_components=True):
    cfg = st["cfg"]
    g = capture(torch, lambda: [run_layer(kc, st, l) for l in range(cfg.n_layers)])
    for _ in range(3):
        g.replay()
    times = time_graph(torch, g, reps)
    del g
    step_ms = mean(times)
    out = {"us_per_layer_step": step_ms * 1e3 / cfg.n_layers, "ms_per_step": step_ms,
           "step_ms_spread": spread(times), "layers": cfg.n_layers, "batch": cfg.batch, "seq_len": cfg.n_ctx,
           "topk": f"{cfg.frac_num}/{cfg.frac_den}"}
    sb = step_bytes_decode(cfg)
    out["layer_step_GBps"] = sb / (step_ms * 1e-3) / 1e9
    out["layer_step_frac_of_hbm"] = out["layer_step_GBps"] / pk["hbm_gbs"]
    if with_components:
        out.update(decode_components(kc, torch, st, reps, pk))
    return out


def time_prefill_stack(kc, torch, st, reps, pk):
    cfg = st["cfg"]
    n = cfg.n_layers
    two_pass, one_pass, gather, sp_flops = prefill_flops(cfg)
    g = capture(torch, lambda: [run_layer(kc, st, l) for l in range(n)])
    g.replay()
    times = time_graph(torch, g, reps)
    del g
    g_sel = capture(torch, lambda: [run_layer(kc, st, l, "select") for l in range(n)])
    sel_ms = mean(time_graph(torch, g_sel, reps)) / len(cfg.anchors)
    del g_sel
    g_attn = capture(torch, lambda: [run_layer(kc, st, l, "attn") for l in range(n)])
    attn_ms = mean(time_graph(torch, g_attn, reps)) / n
    del g_attn
    tf = two_pass / (sel_ms * 1e-3) / 1e12
    sp_tf = sp_flops / (attn_ms * 1e-3) / 1e12
    return {"ms_per_layer": mean(times) / n, "ms_per_step": mean(times), "step_ms_spread": spread(times),
            "layers": n, "anchors": list(cfg.anchors), "seq_len": cfg.n_ctx,
            "topk": f"{cfg.frac_num}/{cfg.frac_den}",
            "anchor_select_ms": sel_ms, "sparse_prefill_ms_per_layer": attn_ms,
            "roofline_anchor_scoring": {"bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"],
                                        "unit": "TFLOP/s", "frac": tf / pk["bf16_tflops"],
                                        "flops": "two-pass executed (exact post-softmax pooling)",
                                        "one_pass_equiv_frac": tf / 2 / pk["bf16_tflops"],
                                        "note": "whole anchor select (score-and-pool + Top-k) time"},
            "roofline_sparse_prefill": {"bound": "tensor", "achieved": sp_tf, "peak": pk["bf16_tflops"],
                                        "unit": "TFLOP/s", "frac": sp_tf / pk["bf16_tflops"],
                                        "flops": sparse_flops_note(),
                                        "gathered_GBps_effective": gather / (attn_ms * 1e-3) / 1e9,
                                        "gathered_bytes": gather,
                                        "note": "gathered rows are mostly served by L2 (tiles of a head share "
                                                "rows), so the tensor pipe, not HBM, bounds this kernel"}}


def sparse_flops_note():
    return "4 x 32 rows x k_t x d per (head, tile): S = Q K_S^T and O = P V_S"


def free(torch, *objs):
    for o in objs:
        if isinstance(o, dict):
            o.clear()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def other_configs(kc, synth, torch, dev, reps, pk):
    """The remaining workloads, one at a time (each freed before the next)."""
    out = {}
    st = build_stack(kc, synth, torch, dev, SMALL_DECODE_CFG)
    r = time_decode_stack(kc, torch, st, max(reps, 20), pk)
    r["note"] = "latency-dominated (0.7 MB per step): the roofline fraction is not meaningful here"
    r["device_error_word"] = st["ws"].error()
    out[SMALL_DECODE_CFG] = r
    free(torch, st)

    st = build_stack(kc, synth, torch, dev, BATCHED_DECODE_CFG)
    r = time_decode_stack(kc, torch, st, reps, pk)
    r["device_error_word"] = st["ws"].error()
    out[BATCHED_DECODE_CFG] = r
    free(torch, st)

    long = {}
    for fr in LONG_PREFILL_FRACS:
        st = build_stack(kc, synth, torch, dev, LONG_PREFILL_CFG, frac=fr)
        r = time_prefill_stack(kc, torch, st, max(2, min(reps, 3)), pk)
        r["device_error_word"] = st["ws"].error()
        long[f"{fr[0]}/{fr[1]}"] = r
        free(torch, st)
    out[LONG_PREFILL_CFG] = long
    return out


def dense_denominators(kc, torch, dec, pre, reps):
    """The library's dense attention (the role FlashAttention-3 plays on the
    pages) on the 32K decode and prefill layers."""
    out = {}
    dcfg = dec["cfg"]
    shape = dec["shape"]
    g = capture(torch, lambda: [kc.dense_ref(shape, *dec["layers"][l], causal=False, o=dec["outs"][l],
                                             ws=dec["ws"]) for l in range(dcfg.n_layers)])
    t = time_graph(torch, g, reps)
    del g
    out[DECODE_CFG] = {"dense_us_per_layer": mean(t) * 1e3 / dcfg.n_layers,
                       "bytes_per_layer": 2 * dcfg.batch * dcfg.hkv * dcfg.n_ctx * dcfg.d * 2}
    if pre is not None:
        pcfg = pre["cfg"]
        q, k, v = pre["layers"][1]
        g = capture(torch, lambda: kc.dense_ref(pre["shape"], q, k, v, causal=True, o=pre["outs"][1],
                                                ws=pre["ws"]))
        t = time_graph(torch, g, 3)
        del g
        flops = 4 * pcfg.hq * pcfg.d * sum(min(32 * (i + 1), pcfg.n_ctx) for i in range(-(-pcfg.n_ctx // 32))) * 32
        out[PREFILL_CFG] = {"dense_causal_ms_per_layer": mean(t), "flops_per_layer": flops,
                            "tflops": flops / (mean(t) * 1e-3) / 1e12}
    torch_sdpa_context(torch, dec, pre, reps, out)
    return out


def torch_sdpa_context(torch, dec, pre, reps, out):
    """For context beside the library's own dense path: PyTorch's
    scaled_dot_product_attention (whatever backend it picks on this device)
    on the same decode layers (grouped query heads) and on one prefill layer
    (causal; K and V expanded to the query heads outside the timed region).
    A library kernel, not this library's path; None where it fails."""
    import torch.nn.functional as F
    dcfg = dec["cfg"]
    try:
        layers = dec["layers"]
        g = capture(torch, lambda: [F.scaled_dot_product_attention(*layers[l], enable_gqa=True)
                                    for l in range(dcfg.n_layers)])
        t = time_graph(torch, g, reps)
        del g
        out[DECODE_CFG]["torch_sdpa_us_per_layer"] = mean(t) * 1e3 / dcfg.n_layers
    except Exception as e:   # noqa: BLE001 - context only
        out[DECODE_CFG]["torch_sdpa_us_per_layer"] = None
        out[DECODE_CFG]["torch_sdpa_error"] = str(e).splitlines()[0][:200]
    if pre is None:
        return
    try:
        q, k, v = pre["layers"][1]
        rep = q.shape[1] // k.shape[1]
        ke, ve = k.repeat_interleave(rep, dim=1), v.repeat_interleave(rep, dim=1)
        g = capture(torch, lambda: F.scaled_dot_product_attention(q, ke, ve, is_causal=True))
        t = time_graph(torch, g, 3)
        del g, ke, ve
        out[PREFILL_CFG]["torch_sdpa_causal_ms_per_layer"] = mean(t)
    except Exception as e:   # noqa: BLE001 - context only
        out[PREFILL_CFG]["torch_sdpa_causal_ms_per_layer"] = None
        out[PREFILL_CFG]["torch_sdpa_error"] = str(e).splitlines()[0][:200]
    torch.cuda.empty_cache()


def run_kascade(args, rank, world, local):
    import torch
    from sparse_attention_long_anchor_b200 import kascade as kc
    from sparse_attention_long_anchor_b200 import synth

    dev = f"cuda:{local}"
    torch.cuda.set_device(local)
    pk = peaks()

    dec = build_stack(kc, synth, torch, dev, DECODE_CFG)
    dcfg = dec["cfg"]
    n_dec = dcfg.n_layers
    g_dec = capture(torch, lambda: [run_layer(kc, dec, l) for l in range(n_dec)])
    pre = build_stack(kc, synth, torch, dev, PREFILL_CFG) if not args.decode_only else None
    g_pre = None
    if pre is not None:
        g_pre = capture(torch, lambda: [run_layer(kc, pre, l) for l in range(pre["cfg"].n_layers)])

    for _ in range(args.warmup):
        g_dec.replay()
        if g_pre is not None:
            g_pre.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for e0, e1, e2 in ev:
        e0.record()
        g_dec.replay()
        e1.record()
        if g_pre is not None:
            g_pre.replay()
        e2.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    dec_steps = [e0.elapsed_time(e1) for e0, e1, _ in ev]
    pre_steps = [e1.elapsed_time(e2) for _, e1, e2 in ev] if g_pre is not None else []
    dec_ms = dist_max(mean(dec_steps), world)
    pre_ms = dist_max(mean(pre_steps), world) if pre_steps else 0.0
    # the decode step's spread over 100 further replays (10 untimed first),
    # apart from the timed steps above
    for _ in range(10):
        g_dec.replay()
    replays_100 = spread(time_graph(torch, g_dec, 100))
    del g_dec, g_pre

    # ---- per-kernel components of the headline stack (CUDA events over
    # graph replays on this stream)
    reps = max(5, args.steps)
    comp = decode_components(kc, torch, dec, reps, pk)
    traffic = profiled_traffic("decode_attn_kernel")
    roofline = {"bound": "hbm", "kernel": "decode_attn_kernel (sparse decode, row a6)",
                "achieved": comp["sparse_decode_GBps"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": comp["sparse_decode_frac_of_hbm"], "traffic": traffic,
                "peak_source": pk["source"] + " hbm_gbs (burst copy)",
                "algorithmic_bytes_per_launch": comp["sparse_decode_algorithmic_bytes"],
                "us_per_launch": comp["sparse_decode_us_per_launch"]}
    sb = step_bytes_decode(dcfg)
    headline = {"us_per_layer_step": dec_ms * 1e3 / n_dec, "ms_per_step": dec_ms, "step_ms_spread": spread(dec_steps),
                "step_ms_spread_100_replays": replays_100,
                "layer_step_GBps": sb / (dec_ms * 1e-3) / 1e9,
                "layer_step_frac_of_hbm": sb / (dec_ms * 1e-3) / 1e9 / pk["hbm_gbs"], **comp}
    # kernels per step, as the library reports them for these shapes on this device
    n_anchor = len(dcfg.anchors)
    launches = n_anchor * (kc.launch_count(dec["shape"], kc.OP_SELECT) + 1) + (n_dec - n_anchor)

    prefill_obj = None
    if pre is not None:
        pcfg = pre["cfg"]
        prefill_obj = time_prefill_stack(kc, torch, pre, 3, pk)
        prefill_obj.update({"workload": PREFILL_CFG, "value": pre_ms / pcfg.n_layers, "unit": "ms/layer",
                            "ms_per_step": pre_ms, "step_ms_spread_timed_loop": spread(pre_steps)})
        n_anchor_pre = len(pcfg.anchors)
        launches += n_anchor_pre * (kc.launch_count(pre["shape"], kc.OP_SELECT) + 1) + (pcfg.n_layers - n_anchor_pre)

    dense = dense_denominators(kc, torch, dec, pre, reps)
    dense[DECODE_CFG]["sparse_us_per_layer_step"] = headline["us_per_layer_step"]
    dense[DECODE_CFG]["speedup"] = dense[DECODE_CFG]["dense_us_per_layer"] / headline["us_per_layer_step"]
    sd = dense[DECODE_CFG].get("torch_sdpa_us_per_layer")
    if sd:
        dense[DECODE_CFG]["speedup_vs_torch_sdpa"] = sd / headline["us_per_layer_step"]
    if pre is not None:
        dense[PREFILL_CFG]["sparse_ms_per_layer"] = prefill_obj["value"]
        dense[PREFILL_CFG]["speedup"] = dense[PREFILL_CFG]["dense_causal_ms_per_layer"] / prefill_obj["value"]
        sp = dense[PREFILL_CFG].get("torch_sdpa_causal_ms_per_layer")
        if sp:
            dense[PREFILL_CFG]["speedup_vs_torch_sdpa"] = sp / prefill_obj["value"]

    # ---- end to end through the public API: the step's queries (every
    # layer's q, one pinned host buffer) copied in, the layers run, the step's
    # outputs copied back; one copy each way
    q_all = torch.stack([dec["layers"][l][0] for l in range(n_dec)])
    o_all = torch.empty_like(q_all)
    host_q = q_all.cpu().pin_memory()
    host_o = torch.empty_like(host_q).pin_memory()
    e2e = dict(dec)
    e2e["layers"] = {l: (q_all[l], dec["layers"][l][1], dec["layers"][l][2]) for l in range(n_dec)}
    e2e["outs"] = {l: o_all[l] for l in range(n_dec)}
    h2d = host_q.numel() * host_q.element_size()
    d2h = host_o.numel() * host_o.element_size()

    def e2e_step():
        q_all.copy_(host_q, non_blocking=True)
        for l in range(n_dec):
            run_layer(kc, e2e, l)
        host_o.copy_(o_all, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        e2e_step()
    t1.record()
    torch.cuda.synchronize()
    e2e_ms = dist_max(t0.elapsed_time(t1) / args.steps, world)

    # prefill end to end through the public API: layer 0's queries copied in
    # from pinned host memory, the 36 layers as eager calls, the last layer's
    # output copied back
    if pre is not None:
        n_pre = pre["cfg"].n_layers
        pq = pre["layers"][0][0]
        po = pre["outs"][n_pre - 1]
        host_pq = pq.cpu().pin_memory()
        host_po = torch.empty(po.shape, dtype=po.dtype, pin_memory=True)

        def e2e_prefill_step():
            pq.copy_(host_pq, non_blocking=True)
            for l in range(n_pre):
                run_layer(kc, pre, l)
            host_po.copy_(po, non_blocking=True)

        e2e_prefill_step()
        torch.cuda.synchronize()
        p_steps = max(1, min(args.steps, 3))
        t0.record()
        for _ in range(p_steps):
            e2e_prefill_step()
        t1.record()
        torch.cuda.synchronize()
        pe2e_ms = dist_max(t0.elapsed_time(t1) / p_steps, world)
        prefill_obj["e2e"] = {"value": pe2e_ms / n_pre, "unit": "ms/layer", "steps": p_steps,
                              "h2d_bytes_per_step": host_pq.numel() * host_pq.element_size(),
                              "d2h_bytes_per_step": host_po.numel() * host_po.element_size(),
                              "path": "eager Python API calls per layer; layer 0's q in and the last layer's o out, "
                                      "one pinned copy each"}
        del host_pq, host_po

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if pre is not None:
            cpu = cpu_baseline_block(dcfg, dec["layers"], dec["plan"], pre["cfg"], pre["layers"], pre["plan"])
        else:
            cpu = cpu_baseline_block(dcfg, dec["layers"], dec["plan"])

    err = dec["ws"].error() | (pre["ws"].error() if pre is not None else 0)
    free(torch, dec, pre or {}, e2e)
    configs = None
    if not args.headline_only:
        configs = other_configs(kc, synth, torch, dev, reps, pk)
    all_configs = {DECODE_CFG: headline}
    if prefill_obj is not None:
        all_configs[PREFILL_CFG] = prefill_obj
    if configs:
        all_configs.update(configs)

    value = dec_ms * 1e3 / (n_dec * world)
    line = {
        "metric": METRIC, "value": value, "unit": "us/layer-step", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dec_ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, planted-salient recipe)",
        "config": {"workload": DECODE_CFG, "global_batch": dcfg.batch * world, "seq_len": dcfg.n_ctx,
                   "layers": n_dec, "anchors": list(dcfg.anchors), "topk": f"{dcfg.frac_num}/{dcfg.frac_den}",
                   "parallelism": f"replicas{world}",
                   "value_definition": "max-over-ranks decode step time / (layers x ranks)",
                   "l2": "inputs larger than L2 (4.3 GB KV per decode step), no flush",
                   "timing": "CUDA graph per stack, CUDA events per step, max over ranks"},
        "step_ms_spread": spread(dec_steps),
        "roofline": roofline, "prefill": prefill_obj, "configs": all_configs, "dense": dense,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_ms * 1e3 / (n_dec * world), "unit": "us/layer-step", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "path": "eager Python API calls per layer; the step's q (all layers) in and o out, one pinned copy each"},
        "gpu_launches": launches * args.steps,
        "device_error_word": err,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("kascade", "reference"), default="kascade")
    ap.add_argument("--decode-only", action="store_true", help="skip the prefill stack")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the other workloads (2K decode, batched 64K decode, 128K prefill)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    rank, world, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_kascade(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
