"""Benchmark of the Kascade hot path on B200.

One step = one decode step of the 32-layer Llama-3.1-8B-shaped stack
(B=1, Hq=32, Hkv=8, d=128, N=32768, Top-k 10 %, anchors {0, 8, 16, 24}) and
one causal prefill of the 36-layer Qwen3-8B-shaped stack (N=32768, tile 32,
anchors {0, 9, 18, 27}), each captured as a CUDA graph.  The headline value is
sparse decode microseconds per layer-step; the prefill figure (ms per layer)
rides along in the same JSON line.

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
import hashlib
import json
import math
import os
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
BATCHED_DECODE_CFG = "decode_llama8b_b8_n64k"


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


def kernel_source_hash(name: str) -> str:
    path = os.path.join(ROOT, "sparse_attention_long_anchor_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(profile: str, source: str):
    """DRAM bytes per launch recorded in a profile summary, or None when the
    kernel source changed after the capture."""
    path = os.path.join(ROOT, "profiles", profile)
    try:
        txt = open(path).read()
    except OSError:
        return None
    vals = {}
    for line in txt.splitlines():
        for key in ("traffic_bytes_per_launch:", "source_sha:"):
            if line.strip().startswith(key):
                vals[key] = line.split(":", 1)[1].strip().strip("`")
    if vals.get("source_sha:") != kernel_source_hash(source):
        return None
    try:
        return float(vals["traffic_bytes_per_launch:"])
    except (KeyError, ValueError):
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


# ----------------------------------------------------------------------------- oracle timing


def oracle_decode_sample(cfg, layers_np, plan, threads_note):
    """Time the oracle on one anchor layer and one reuse layer of the decode
    stack; returns (us per layer-step weighted like the stack, detail)."""
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
    return per_layer * 1e6, {"anchor_layer_s": anchor_s, "reuse_layer_s": reuse_s}


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


# ----------------------------------------------------------------------------- reference arm


def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores on bounded samples of
    the decode workload (one anchor + one reuse layer per step)."""
    if rank != 0:
        return
    import numpy as np
    from sparse_attention_long_anchor_b200 import synth
    cfg = synth.CONFIGS[DECODE_CFG]
    plan, layers = synth.make_stack(cfg, device="cpu", layers=[0, 1])
    L = [host_copy_layer(*layers[0]), host_copy_layer(*layers[1])]
    vals = []
    for step in range(args.warmup + args.steps):
        v, _ = oracle_decode_sample(cfg, L, plan, None)
        if step >= args.warmup:
            vals.append(v)
    value = float(np.mean(vals))
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "us/layer-step", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": value * cfg.n_layers / 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": DECODE_CFG, "global_batch": cfg.batch, "seq_len": cfg.n_ctx, "layers": cfg.n_layers,
                   "parallelism": f"replicas{world}"},
        "cpu_baseline": {"value": value, "unit": "us/layer-step", "cores": cores, "kind": "oracle",
                         "sample": "per step: oracle on anchor layer 0 and reuse layer 1 of the stack, weighted "
                                   "4 anchor : 28 reuse layers"},
        "e2e": {"value": value, "unit": "us/layer-step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- kascade arm


def build_decode(kc, synth, torch, dev):
    cfg = synth.CONFIGS[DECODE_CFG]
    plan, layers = synth.make_stack(cfg, device=dev)
    frac = (cfg.frac_num, cfg.frac_den)
    shape = kc.Shape.make(cfg.batch, cfg.hq, cfg.hkv, cfg.d, 1, cfg.n_ctx, frac, flags=kc.FLAG_PDL)
    ws = kc.Workspace(shape, device=dev)
    idx = {a: torch.empty(kc.index_count(shape), dtype=torch.int32, device=dev) for a in cfg.anchors}
    hms = {l: torch.tensor(p[2], dtype=torch.int32, device=dev) for l, p in enumerate(plan) if not p[0]}
    outs = {l: torch.empty_like(layers[l][0]) for l in range(cfg.n_layers)}
    return cfg, plan, layers, shape, ws, idx, hms, outs


def decode_layer(kc, st, l, which="all"):
    """One decode layer.  Kernels use programmatic dependent launch; a reuse
    layer reads an index set written at least two launches earlier and a KV
    cache that no kernel of the step writes, so its gathers may start early."""
    cfg, plan, layers, shape, ws, idx, hms, outs = st
    is_anchor, anchor, _ = plan[l]
    q, k, v = layers[l]
    if is_anchor:
        if which in ("all", "select"):
            kc.select(shape, q, k, idx[l], ws=ws)
        if which in ("all", "attn"):
            kc.sparse_decode(shape, q, k, v, idx[l], None, o=outs[l], ws=ws)
    elif which in ("all", "attn"):
        kc.sparse_decode(_stable_shape(kc, shape), q, k, v, idx[anchor], hms[l], o=outs[l], ws=ws)


_STABLE = {}


def _stable_shape(kc, shape):
    """The reuse layers' shape (early gathers), built once per stack shape."""
    hit = _STABLE.get(id(shape))
    if hit is None or hit[0] is not shape:
        hit = _STABLE[id(shape)] = (shape, shape.with_flags(kc.FLAG_PDL | kc.FLAG_INPUTS_STABLE))
    return hit[1]


def build_prefill(kc, synth, torch, dev):
    cfg = synth.CONFIGS[PREFILL_CFG]
    plan, layers = synth.make_stack(cfg, device=dev)
    frac = (cfg.frac_num, cfg.frac_den)
    shape = kc.Shape.make(cfg.batch, cfg.hq, cfg.hkv, cfg.d, cfg.n_ctx, cfg.n_ctx, frac, flags=kc.FLAG_PDL)
    ws = kc.Workspace(shape, device=dev)
    idx = {a: torch.empty(kc.index_count(shape), dtype=torch.int32, device=dev) for a in cfg.anchors}
    hms = {l: torch.tensor(p[2], dtype=torch.int32, device=dev) for l, p in enumerate(plan) if not p[0]}
    outs = {l: torch.empty_like(layers[l][0]) for l in range(cfg.n_layers)}
    return cfg, plan, layers, shape, ws, idx, hms, outs


def prefill_layer(kc, st, l, which="all"):
    cfg, plan, layers, shape, ws, idx, hms, outs = st
    is_anchor, anchor, _ = plan[l]
    q, k, v = layers[l]
    if is_anchor:
        if which in ("all", "select"):
            kc.select(shape, q, k, idx[l], ws=ws)
        if which in ("all", "attn"):
            kc.sparse_prefill(shape, q, k, v, idx[l], None, o=outs[l], ws=ws)
    elif which in ("all", "attn"):
        kc.sparse_prefill(shape, q, k, v, idx[anchor], hms[l], o=outs[l], ws=ws)


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
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    g.replay()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def decode_bytes(cfg):
    kk = math.ceil(cfg.frac_num * cfg.n_ctx / cfg.frac_den)
    reuse = cfg.batch * cfg.hkv * (2 * kk * cfg.d * 2 + 4 * kk)
    anchor_score = cfg.batch * cfg.hkv * cfg.n_ctx * cfg.d * 2
    return kk, reuse, anchor_score


def batched_decode_component(kc, synth, torch, dev, reps, pk):
    """Anchor select and sparse decode of the batched 64K decode stack (B=8,
    N=65536, 10 %), where a reuse layer gathers 216 MB: the bandwidth-bound
    regime of the sparse decode.  Layers 0 (anchor), 1 and 2 (reuse) are
    built; the timed graph alternates the two reuse layers, so the 432 MB
    they gather together exceed L2."""
    cfg = synth.CONFIGS[BATCHED_DECODE_CFG]
    plan, layers = synth.make_stack(cfg, device=dev, layers=[0, 1, 2])
    frac = (cfg.frac_num, cfg.frac_den)
    shape = kc.Shape.make(cfg.batch, cfg.hq, cfg.hkv, cfg.d, 1, cfg.n_ctx, frac, flags=kc.FLAG_PDL)
    stable = shape.with_flags(kc.FLAG_PDL | kc.FLAG_INPUTS_STABLE)
    ws = kc.Workspace(shape, device=dev)
    idx = torch.empty(kc.index_count(shape), dtype=torch.int32, device=dev)
    q0, k0, _ = layers[0]
    hms = {l: torch.tensor(plan[l][2], dtype=torch.int32, device=dev) for l in (1, 2)}
    outs = {l: torch.empty_like(layers[l][0]) for l in (1, 2)}
    kc.select(shape, q0, k0, idx, ws=ws)
    torch.cuda.synchronize()

    def reuse(l):
        q, k, v = layers[l]
        kc.sparse_decode(stable, q, k, v, idx, hms[l], o=outs[l], ws=ws)

    g_sel = capture(torch, lambda: kc.select(shape, q0, k0, idx, ws=ws))
    g_att = capture(torch, lambda: [reuse(1 + (i & 1)) for i in range(8)])
    sel_us = time_graph(torch, g_sel, reps) * 1e3
    att_us = time_graph(torch, g_att, reps) * 1e3 / 8
    _, reuse_bytes, score_bytes = decode_bytes(cfg)
    gbs = reuse_bytes / (att_us * 1e-6) / 1e9
    err = ws.error()
    del g_sel, g_att
    return {"workload": BATCHED_DECODE_CFG, "sparse_decode_us": att_us, "algorithmic_bytes": reuse_bytes,
            "sparse_decode_GBps": gbs, "frac_of_hbm": gbs / pk["hbm_gbs"],
            "anchor_select_us": sel_us, "anchor_select_GBps_on_K": score_bytes / (sel_us * 1e-6) / 1e9,
            "device_error_word": err}


def prefill_flops(cfg):
    """Executed flops of the two-pass exact scoring of one anchor layer and
    gathered bytes / flops of one sparse prefill layer."""
    T = math.ceil(cfg.n_ctx / cfg.tile)
    e = [min(cfg.tile * (t + 1), cfg.n_ctx) for t in range(T)]
    kt = [math.ceil(cfg.frac_num * x / cfg.frac_den) for x in e]
    one_pass = sum(2 * cfg.hq * cfg.d * cfg.tile * x for x in e)
    gather = sum(cfg.batch * cfg.hkv * 2 * k * cfg.d * 2 for k in kt)
    sparse_flops = sum(cfg.batch * cfg.hq * 4 * cfg.tile * k * cfg.d for k in kt)
    return 2 * one_pass, one_pass, gather, sparse_flops


def run_kascade(args, rank, world, local):
    import numpy as np
    import torch
    from sparse_attention_long_anchor_b200 import kascade as kc
    from sparse_attention_long_anchor_b200 import synth

    dev = f"cuda:{local}"
    torch.cuda.set_device(local)
    pk = peaks()

    dec = build_decode(kc, synth, torch, dev)
    dcfg = dec[0]
    n_dec = dcfg.n_layers
    g_dec = capture(torch, lambda: [decode_layer(kc, dec, l) for l in range(n_dec)])
    pre = build_prefill(kc, synth, torch, dev) if not args.decode_only else None
    g_pre = None
    if pre is not None:
        pcfg = pre[0]
        g_pre = capture(torch, lambda: [prefill_layer(kc, pre, l) for l in range(pcfg.n_layers)])

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
    dec_ms = sum(e0.elapsed_time(e1) for e0, e1, _ in ev) / args.steps
    pre_ms = sum(e1.elapsed_time(e2) for _, e1, e2 in ev) / args.steps if g_pre is not None else 0.0
    dec_ms = dist_max(dec_ms, world)
    pre_ms = dist_max(pre_ms, world)

    # ---- per-kernel components (CUDA events over graph replays on this stream)
    kk, reuse_bytes, anchor_score_bytes = decode_bytes(dcfg)
    g_attn = capture(torch, lambda: [decode_layer(kc, dec, l, "attn") for l in range(n_dec)])
    g_sel = capture(torch, lambda: [decode_layer(kc, dec, l, "select") for l in range(n_dec)])
    reps = max(5, args.steps)
    attn_ms = time_graph(torch, g_attn, reps)          # 32 sparse-decode launches
    sel_ms = time_graph(torch, g_sel, reps)            # 4 x (scoring + select)
    attn_us_per_launch = attn_ms * 1e3 / n_dec
    n_anchor = len(dcfg.anchors)
    attn_gbs = reuse_bytes / (attn_us_per_launch * 1e-6) / 1e9
    traffic = profiled_traffic("decode_attn_llama8b_n32k.md", "decode_attn.cu")
    roofline = {"bound": "hbm", "kernel": "decode_attn_kernel (sparse decode, row a6)",
                "achieved": attn_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": attn_gbs / pk["hbm_gbs"],
                "traffic": traffic, "peak_source": pk["source"] + " hbm_gbs (burst copy)",
                "algorithmic_bytes_per_launch": reuse_bytes, "us_per_launch": attn_us_per_launch}
    components = {"sparse_decode_us_per_layer": attn_us_per_launch,
                  "anchor_select_us_per_anchor": sel_ms * 1e3 / n_anchor,
                  "anchor_scoring_bytes": anchor_score_bytes,
                  "anchor_select_GBps_on_K": anchor_score_bytes / (sel_ms * 1e-3 / n_anchor) / 1e9}
    if args.batched_decode:
        components["batched_decode"] = batched_decode_component(kc, synth, torch, dev, reps, pk)
    # kernels per step, as the library reports them for these shapes on this device
    launches = n_anchor * (kc.launch_count(dec[3], kc.OP_SELECT) + 1) + (n_dec - n_anchor)

    prefill_obj = None
    if g_pre is not None:
        pcfg = pre[0]
        two_pass, one_pass, gather, sp_flops = prefill_flops(pcfg)
        gp_sel = capture(torch, lambda: [prefill_layer(kc, pre, l, "select") for l in range(pcfg.n_layers)])
        gp_attn = capture(torch, lambda: [prefill_layer(kc, pre, l, "attn") for l in range(pcfg.n_layers)])
        psel_ms = time_graph(torch, gp_sel, 3) / len(pcfg.anchors)
        pattn_ms = time_graph(torch, gp_attn, 3) / pcfg.n_layers
        tf = two_pass / (psel_ms * 1e-3) / 1e12
        prefill_obj = {
            "workload": PREFILL_CFG, "value": pre_ms / pcfg.n_layers, "unit": "ms/layer",
            "ms_per_step": pre_ms, "layers": pcfg.n_layers, "anchors": list(pcfg.anchors),
            "anchor_select_ms": psel_ms, "sparse_prefill_ms_per_layer": pattn_ms,
            "roofline_anchor_scoring": {"bound": "tensor", "achieved": tf, "peak": pk["bf16_tflops"],
                                        "unit": "TFLOP/s", "frac": tf / pk["bf16_tflops"],
                                        "flops": "two-pass executed", "one_pass_equiv_frac":
                                        tf / 2 / pk["bf16_tflops"],
                                        "note": "whole anchor select (score-and-pool + Top-k) time"},
            "roofline_sparse_prefill": {"bound": "hbm", "achieved": gather / (pattn_ms * 1e-3) / 1e9,
                                        "peak": pk["hbm_gbs"], "unit": "GB/s (gathered rows, effective)",
                                        "frac": gather / (pattn_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                                        "tensor_tflops": sp_flops / (pattn_ms * 1e-3) / 1e12},
        }
        launches += len(pcfg.anchors) * (kc.launch_count(pre[3], kc.OP_SELECT) + 1) + (pcfg.n_layers - len(pcfg.anchors))

    # ---- end to end through the public API: the step's queries (every layer's
    # q, one pinned host buffer) copied in, the layers run, the step's outputs
    # copied back; one copy each way
    cfg, plan, layers, shape, ws, idx, hms, outs = dec
    q_all = torch.stack([layers[l][0] for l in range(n_dec)])
    o_all = torch.empty_like(q_all)
    host_q = q_all.cpu().pin_memory()
    host_o = torch.empty_like(host_q).pin_memory()
    e2e_dec = (cfg, plan, [(q_all[l], layers[l][1], layers[l][2]) for l in range(n_dec)], shape, ws, idx, hms,
               {l: o_all[l] for l in range(n_dec)})
    h2d = host_q.numel() * host_q.element_size()
    d2h = host_o.numel() * host_o.element_size()

    def e2e_step():
        q_all.copy_(host_q, non_blocking=True)
        for l in range(n_dec):
            decode_layer(kc, e2e_dec, l)
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

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        L = [host_copy_layer(*layers[0]), host_copy_layer(*layers[1])]
        v, detail = oracle_decode_sample(cfg, L, plan, None)
        cpu = {"value": v, "unit": "us/layer-step", "cores": blas_threads(), "kind": "oracle",
               "sample": "oracle (fp64 numpy) on anchor layer 0 and reuse layer 1 of this stack, weighted "
                         "4 anchor : 28 reuse layers; " + json.dumps({k: round(x, 3) for k, x in detail.items()})}

    value = dec_ms * 1e3 / (n_dec * world)
    line = {
        "metric": METRIC, "value": value, "unit": "us/layer-step", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dec_ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded, planted-salient recipe)",
        "config": {"workload": DECODE_CFG, "global_batch": dcfg.batch * world, "seq_len": dcfg.n_ctx,
                   "layers": n_dec, "anchors": list(dcfg.anchors), "topk": f"{dcfg.frac_num}/{dcfg.frac_den}",
                   "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (4.3 GB KV per decode step), no flush",
                   "timing": "CUDA graph per stack, CUDA events, max over ranks"},
        "roofline": roofline, "components": components, "prefill": prefill_obj,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_ms * 1e3 / (n_dec * world), "unit": "us/layer-step", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "path": "eager Python API calls per layer; the step's q (all layers) in and o out, one pinned copy each"},
        "gpu_launches": launches * args.steps,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g_dec, g_pre


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("kascade", "reference"), default="kascade")
    ap.add_argument("--decode-only", action="store_true", help="skip the prefill stack")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batched-decode", action="store_true",
                    help="also time the batched 64K decode (B=8) select and sparse decode, outside the step")
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
