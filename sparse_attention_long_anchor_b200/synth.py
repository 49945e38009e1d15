"""Seeded synthetic inputs and layer plans for the Kascade workloads.

This module draws random tensors and holds the workload shapes; it contains
none of the attention arithmetic.  Both the CUDA path (tests, bench) and the
oracle checks use these inputs, so it has no dependency on either.

Input recipe (a reading of the Kascade README's Abstract, which motivates the
method with sparse post-softmax attention whose heavy keys drift slowly from
layer to layer; the page gives no distribution):

* Q, K, V ~ N(0, 1), rounded once to bf16 after the plants below are added;
* per (layer, batch, kv head h): a random unit vector u; 64 "salient" key
  positions drawn without replacement from [1, N) get K += 4u; the sink key 0
  gets K += 8u; every query row of h's G query heads gets Q += 2u;
* drift: in a reuse layer the salient set of head h is the previous layer's
  set of head head_map[h] with 6 of its 64 positions replaced by fresh ones;
* prefill band: per (layer, batch, kv head) random unit vectors w_c for the
  256-key buckets c = j // 256; K_j += 3 w_c(j) and Q_i += 1.5 (w_c(i) +
  w_c(i)-1), which boosts a diagonal-local band of 256-512 keys;
* head_map of a reuse layer: uniform with replacement over the kv heads.
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["StackConfig", "CONFIGS", "layer_plan", "salient_sets", "make_layer", "make_stack",
           "new_generator", "kv_bytes", "n_tiles"]


@dataclasses.dataclass(frozen=True)
class StackConfig:
    name: str
    mode: str               # "decode" or "prefill"
    batch: int
    hq: int
    hkv: int
    d: int
    n_ctx: int
    n_layers: int
    anchors: tuple
    frac_num: int = 10
    frac_den: int = 100
    tile: int = 32
    head_map: str = "random"   # "identity" or "random"
    drift: bool = True
    band: bool = False
    n_salient: int = 64
    seed: int = 0

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def q_len(self) -> int:
        return 1 if self.mode == "decode" else self.n_ctx

    def with_(self, **kw) -> "StackConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    # decode, 1 anchor + 1 reuse layer, identity head_map
    "decode_b1_h8_n2k": StackConfig("decode_b1_h8_n2k", "decode", 1, 8, 2, 64, 2048, 2, (0,),
                                    head_map="identity", drift=False),
    # decode, Llama-3.1-8B-shaped 32-layer stack
    "decode_llama8b_n32k": StackConfig("decode_llama8b_n32k", "decode", 1, 32, 8, 128, 32768, 32,
                                       (0, 8, 16, 24)),
    # batched decode, 8 sequences of 64K
    "decode_llama8b_b8_n64k": StackConfig("decode_llama8b_b8_n64k", "decode", 8, 32, 8, 128, 65536, 32,
                                          (0, 8, 16, 24)),
    # causal prefill, Qwen3-8B-shaped 36-layer stack
    "prefill_qwen8b_n32k": StackConfig("prefill_qwen8b_n32k", "prefill", 1, 32, 8, 128, 32768, 36,
                                       (0, 9, 18, 27), band=True),
    # long causal prefill, 1 anchor + 7 reuse layers (frac swept 5/10/20 %)
    "prefill_n128k": StackConfig("prefill_n128k", "prefill", 1, 32, 8, 128, 131072, 8, (0,), band=True),
}


def layer_plan(cfg: StackConfig):
    """For each layer: (is_anchor, anchor layer it reads, head_map list).

    A reuse layer reads the index sets of the nearest preceding anchor."""
    gen = torch.Generator().manual_seed(cfg.seed * 7919 + 17)
    plan = []
    last_anchor = None
    for layer in range(cfg.n_layers):
        if layer in cfg.anchors or last_anchor is None:
            last_anchor = layer
            plan.append((True, layer, list(range(cfg.hkv))))
            continue
        if cfg.head_map == "identity":
            hm = list(range(cfg.hkv))
        else:
            hm = torch.randint(0, cfg.hkv, (cfg.hkv,), generator=gen).tolist()
        plan.append((False, last_anchor, hm))
    return plan


def new_generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _sub_seed(cfg_seed: int, layer: int, tag: int) -> int:
    return (cfg_seed * 1_000_003 + layer * 7_919 + tag * 104_729) % (2 ** 62)


def _unit(gen, d, device):
    u = torch.randn(d, generator=gen, device=device, dtype=torch.float32)
    return u / u.norm()


def _fresh_salient(gen, n_ctx, count, exclude=None):
    """`count` distinct positions in [1, n_ctx) not in `exclude` (CPU)."""
    if n_ctx <= 1 or count <= 0:
        return torch.zeros(0, dtype=torch.long)
    perm = torch.randperm(n_ctx - 1, generator=gen) + 1
    if exclude is not None and exclude.numel() > 0:
        perm = perm[~torch.isin(perm, exclude)]
    return perm[:count]


def salient_sets(cfg: StackConfig, plan=None):
    """Salient key positions of every layer: list of [B, Hkv, n_sal] tensors.

    Drawn on the CPU from their own seeded stream, so they do not depend on
    the device the tensors are generated on."""
    plan = layer_plan(cfg) if plan is None else plan
    n = cfg.n_ctx
    n_sal = min(cfg.n_salient, max(n - 1, 0))
    n_swap = max(1, (n_sal * 10 + 99) // 100) if n_sal > 0 else 0   # 10 % drift (6 of 64)
    out = []
    prev = None
    for layer in range(cfg.n_layers):
        gen = torch.Generator().manual_seed(_sub_seed(cfg.seed, layer, 2))
        is_anchor, _, hm = plan[layer]
        cur = torch.zeros(cfg.batch, cfg.hkv, n_sal, dtype=torch.long)
        for b in range(cfg.batch):
            for h in range(cfg.hkv):
                if prev is not None and cfg.drift and not is_anchor and n_sal > 0:
                    src = prev[b, hm[h]]
                    keep = src[torch.randperm(n_sal, generator=gen)[: n_sal - n_swap]]
                    sal = torch.cat([keep, _fresh_salient(gen, n, n_swap, exclude=keep)])
                else:
                    sal = _fresh_salient(gen, n, n_sal)
                cur[b, h, : sal.numel()] = sal
        out.append(cur)
        prev = cur
    return out


def make_layer(cfg: StackConfig, layer: int, salient, device="cpu"):
    """Q, K, V (bf16) of one layer, given that layer's salient sets."""
    gen = new_generator(device, _sub_seed(cfg.seed, layer, 1))
    pgen = torch.Generator().manual_seed(_sub_seed(cfg.seed, layer, 3))
    bsz, hq, hkv, d, n = cfg.batch, cfg.hq, cfg.hkv, cfg.d, cfg.n_ctx
    g_size = cfg.group
    lq = cfg.q_len
    q = torch.randn(bsz, hq, lq, d, generator=gen, device=device, dtype=torch.float32)
    k = torch.randn(bsz, hkv, n, d, generator=gen, device=device, dtype=torch.float32)
    v = torch.randn(bsz, hkv, n, d, generator=gen, device=device, dtype=torch.float32)
    for b in range(bsz):
        for h in range(hkv):
            u = _unit(pgen, d, "cpu").to(device)
            sal = salient[b, h].to(device)
            if sal.numel():
                k[b, h, sal] += 4.0 * u
            k[b, h, 0] += 8.0 * u
            q[b, h * g_size:(h + 1) * g_size] += 2.0 * u
            if cfg.band:
                n_bkt = -(-n // 256)
                w = torch.randn(n_bkt, d, generator=pgen, dtype=torch.float32)
                w = (w / w.norm(dim=1, keepdim=True)).to(device)
                bkt = torch.arange(n, device=device) // 256
                k[b, h] += 3.0 * w[bkt]
                if lq == n:
                    prev = torch.cat([torch.zeros(1, d, device=device), w[:-1]], 0)
                    q[b, h * g_size:(h + 1) * g_size] += 1.5 * (w[bkt] + prev[bkt])
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def make_stack(cfg: StackConfig, device="cpu", layers=None):
    """(plan, {layer: (q, k, v)}) for the listed layers (default: all)."""
    plan = layer_plan(cfg)
    sal = salient_sets(cfg, plan)
    want = range(cfg.n_layers) if layers is None else layers
    return plan, {layer: make_layer(cfg, layer, sal[layer], device) for layer in want}


def kv_bytes(cfg: StackConfig) -> int:
    return 2 * cfg.batch * cfg.hkv * cfg.n_ctx * cfg.d * 2 * cfg.n_layers


def n_tiles(cfg: StackConfig) -> int:
    return math.ceil(cfg.n_ctx / cfg.tile)
