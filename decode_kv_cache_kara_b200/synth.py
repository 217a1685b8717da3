"""Seeded synthetic workloads: paged KV caches, window queries, decode queries.

This module draws random inputs and lays them out; it holds none of the method's arithmetic.
Both the CUDA library and the CPU oracle take their inputs from here.

Value recipe (the pages' workloads are reasoning-model caches; no dataset is used):

* K, V, decode queries: bf16 of N(0, 1) draws (round-to-nearest-even from fp32).
* Heavy keys: runs of consecutive slots, start uniform, length uniform in [run_lo, run_hi],
  until the target fraction of the region is covered; K rows of those slots (every KV head,
  every layer) are multiplied by ``heavy_scale`` (a power of two, so bf16 stays exact).
* Window queries: either N(0, 1) ("normal"), or "neighbour": q for window position i and query
  head h = the K row of the previous slot for h's KV head plus 0.5 * N(0, 1) (position 0 uses
  its own slot).
* Contexts: fixed, or uniform integers in [ctx_lo, ctx_hi] (ragged, unaligned windows).
* Block ids: a seeded permutation; each sequence takes consecutive entries of it, the rest
  forms the free list (stack) in permutation order, so tables are non-contiguous.

Random draws use numpy's PCG64 for the small host-side structure and a torch.Generator on the
target device for the tensors, both seeded from ``seed``.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch

PAGE = 16


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    layers: int
    hq: int
    hkv: int
    head_dim: int
    ctx_lo: int
    ctx_hi: int
    window: int
    keep: int
    page: int = PAGE
    heavy_frac: float = 0.0
    heavy_scale: float = 4.0
    run_lo: int = 2
    run_hi: int = 8
    heavy_where: str = "all"      # "all" slots of the context, or only the "window"
    q_mode: str = "normal"        # "normal" or "neighbour"
    anchor_frac: float = 0.5
    gap_limit: int = 8
    widen: int = 1
    spare_blocks: int = 0         # extra free blocks beyond what one compaction needs
    extra: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads: tiny (the parity case), one 7B-class layer, a 28-layer step with ragged
# contexts, an 8B-class GQA model and the LaCache workload; each line states its sizes.
WORKLOADS = {
    # 1 sequence, 4q/2kv heads, d=64, 512-token cache, window 128, keep 32, 5 % heavy window keys
    "tiny": Workload("tiny", batch=1, layers=1, hq=4, hkv=2, head_dim=64, ctx_lo=512, ctx_hi=512,
                     window=128, keep=32, heavy_frac=0.05, run_lo=2, run_hi=8,
                     heavy_where="window", q_mode="normal", spare_blocks=8),
    # one 7B-class layer: batch 32, 28q/4kv, d=128, 4096-token caches, window 1024, keep 204
    "layer": Workload("layer", batch=32, layers=1, hq=28, hkv=4, head_dim=128, ctx_lo=4096,
                      ctx_hi=4096, window=1024, keep=204, heavy_frac=0.03, run_lo=2, run_hi=16,
                      q_mode="neighbour", spare_blocks=64),
    # full 28-layer step: batch 128, ragged 2K-16K, window 1024, 20 % keep, gap 8, anchors 50 %
    "step": Workload("step", batch=128, layers=28, hq=28, hkv=4, head_dim=128, ctx_lo=2048,
                     ctx_hi=16384, window=1024, keep=204, heavy_frac=0.03, run_lo=2, run_hi=16,
                     q_mode="neighbour", spare_blocks=256),
    # 8B-class GQA: batch 256, 32 layers, 32q/8kv, ragged 8K-32K, window 2048, keep 409
    "gqa8b": Workload("gqa8b", batch=256, layers=32, hq=32, hkv=8, head_dim=128, ctx_lo=8192,
                      ctx_hi=32768, window=2048, keep=409, heavy_frac=0.03, run_lo=2,
                      run_hi=16, q_mode="neighbour", spare_blocks=512),
    # LaCache ladder: batch 8, 32 layers, 8 kv heads, 64K tokens, S=8, O=4, budget 8192, rung 64
    "lacache": Workload("lacache", batch=8, layers=32, hq=32, hkv=8, head_dim=128, ctx_lo=65536,
                        ctx_hi=65536, window=0, keep=0, heavy_frac=0.03, run_lo=2, run_hi=16,
                        spare_blocks=0,
                        extra={"span": 8, "overlap": 4, "budget": 8192, "rung": 64,
                               "sink": 0, "recent": 0, "passes": 3, "refill": 24576}),
}


def _heavy_slots(rng: np.random.Generator, lo: int, hi: int, frac: float, run_lo: int,
                 run_hi: int) -> np.ndarray:
    """Slots in [lo, hi) covered by heavy runs, until round(frac * (hi-lo)) are covered."""
    length = hi - lo
    target = int(round(frac * length))
    mark = np.zeros(length, dtype=bool)
    guard = 0
    while mark.sum() < target and guard < 100000:
        start = int(rng.integers(0, length))
        run = int(rng.integers(run_lo, run_hi + 1))
        mark[start:min(length, start + run)] = True
        guard += 1
    return lo + np.nonzero(mark)[0]


def fresh_blocks_needed(wl: Workload) -> int:
    """Free blocks one compaction of every sequence can pop (upper bound)."""
    if wl.name == "lacache" or wl.extra.get("budget"):
        return wl.batch * math.ceil(wl.extra["budget"] / wl.page)
    return wl.batch * math.ceil((wl.page - 1 + wl.keep) / wl.page)


@torch.no_grad()
def make_cache(wl: Workload, seed: int, device="cpu", layers: int | None = None,
               with_queries: bool = True, dtype=torch.bfloat16, extra_pages: int = 0) -> dict:
    """Build one seeded paged cache for a workload.

    Returns a dict with ``k``/``v`` (lists, one [num_blocks, page, Hkv, d] tensor per layer),
    ``block_table`` [B, max_blocks] int32 (-1 = no block), ``ctx_len`` [B] int32,
    ``free_list`` [num_blocks] int32, ``free_top`` [1] int32, and when ``with_queries`` the
    window queries ``q_win`` (list per layer of [B, W, Hq, d]) and decode queries ``q_dec``
    [B, Hq, d]. Layers default to ``wl.layers``. ``extra_pages`` adds that many table
    columns per sequence and as many spare blocks per sequence, room for a decode loop.
    """
    device = torch.device(device)
    nlayers = wl.layers if layers is None else layers
    rng = np.random.default_rng(np.random.PCG64(seed))
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)

    if wl.ctx_lo == wl.ctx_hi:
        ctx = np.full(wl.batch, wl.ctx_lo, dtype=np.int64)
    else:
        ctx = rng.integers(wl.ctx_lo, wl.ctx_hi + 1, size=wl.batch)
    pages = [math.ceil(int(n) / wl.page) for n in ctx]
    max_blocks = max(pages) + 1 + extra_pages
    num_blocks = sum(pages) + fresh_blocks_needed(wl) + wl.spare_blocks + wl.batch * extra_pages
    perm = rng.permutation(num_blocks).astype(np.int64)

    table = np.full((wl.batch, max_blocks), -1, dtype=np.int32)
    pos = 0
    for b, np_ in enumerate(pages):
        table[b, :np_] = perm[pos:pos + np_]
        pos += np_
    free = np.zeros(num_blocks, dtype=np.int32)
    free_ids = perm[pos:]
    free[:len(free_ids)] = free_ids

    heavy = []
    for b in range(wl.batch):
        n = int(ctx[b])
        lo = n - wl.window if wl.heavy_where == "window" else 0
        heavy.append(_heavy_slots(rng, lo, n, wl.heavy_frac, wl.run_lo, wl.run_hi)
                     if wl.heavy_frac > 0 else np.zeros(0, dtype=np.int64))
    hb = np.concatenate([table[b, s // wl.page] for b, s in enumerate(heavy)]) if heavy else []
    hr = np.concatenate([s % wl.page for s in heavy]) if heavy else []
    hb_t = torch.as_tensor(np.asarray(hb, dtype=np.int64), device=device)
    hr_t = torch.as_tensor(np.asarray(hr, dtype=np.int64), device=device)

    shape = (num_blocks, wl.page, wl.hkv, wl.head_dim)
    ks, vs = [], []
    for _ in range(nlayers):
        k = torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(dtype)
        if hb_t.numel():
            k[hb_t, hr_t] = k[hb_t, hr_t] * wl.heavy_scale
        v = torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(dtype)
        ks.append(k)
        vs.append(v)

    out = {
        "k": ks, "v": vs,
        "block_table": torch.as_tensor(table, device=device),
        "ctx_len": torch.as_tensor(ctx.astype(np.int32), device=device),
        "free_list": torch.as_tensor(free, device=device),
        "free_top": torch.tensor([len(free_ids)], dtype=torch.int32, device=device),
        "num_blocks": num_blocks, "max_blocks": max_blocks, "seed": seed, "workload": wl,
    }
    if with_queries and wl.window > 0:
        out["q_win"] = [make_window_queries(wl, out, ks[i], gen) for i in range(nlayers)]
    if with_queries:
        out["q_dec"] = torch.randn((wl.batch, wl.hq, wl.head_dim), generator=gen, device=device,
                                   dtype=torch.float32).to(dtype)
    return out


@torch.no_grad()
def decode_step_inputs(wl: Workload, seed: int, step: int, layers: int | None = None,
                       dtype=torch.bfloat16) -> list:
    """Seeded inputs of decode step ``step`` (CPU tensors), one dict per layer: the new
    token's ``k`` and ``v`` [B, Hkv, d] ~ N(0, 1) and its query ``q`` [B, Hq, d], each query
    head the new key of its KV head plus N(0, 0.5^2) noise (so the window queries resemble
    the window keys, as in the window-query recipe)."""
    nlayers = wl.layers if layers is None else layers
    gen = torch.Generator()
    gen.manual_seed(seed * 1_000_003 + step)
    out = []
    for _ in range(nlayers):
        k = torch.randn((wl.batch, wl.hkv, wl.head_dim), generator=gen)
        v = torch.randn((wl.batch, wl.hkv, wl.head_dim), generator=gen)
        noise = torch.randn((wl.batch, wl.hq, wl.head_dim), generator=gen)
        q = k.repeat_interleave(wl.group, dim=1) + 0.5 * noise
        out.append({"q": q.to(dtype), "k": k.to(dtype), "v": v.to(dtype)})
    return out


@torch.no_grad()
def make_window_queries(wl: Workload, cache: dict, k_pool: torch.Tensor,
                        gen: torch.Generator) -> torch.Tensor:
    """Window queries [B, W, Hq, d] for one layer (see the module docstring)."""
    device = k_pool.device
    noise = torch.randn((wl.batch, wl.window, wl.hq, wl.head_dim), generator=gen, device=device,
                        dtype=torch.float32)
    if wl.q_mode == "normal":
        return noise.to(k_pool.dtype)
    table = cache["block_table"].long()
    ctx = cache["ctx_len"].long()
    i = torch.arange(wl.window, device=device)
    start = (ctx - wl.window)[:, None]
    nb_slot = start + torch.clamp(i - 1, min=0)[None, :]                      # [B, W]
    blocks = torch.gather(table, 1, nb_slot // wl.page)
    rows = nb_slot % wl.page
    k_nb = k_pool[blocks, rows].float()                                        # [B, W, Hkv, d]
    k_nb = k_nb.repeat_interleave(wl.group, dim=2)                             # [B, W, Hq, d]
    return (k_nb + 0.5 * noise).to(k_pool.dtype)


def random_keep(rng: np.random.Generator, rows: int, window: int, k: int) -> np.ndarray:
    """Arbitrary ascending keep lists [rows, k] (for testing compaction on its own)."""
    out = np.empty((rows, k), dtype=np.int32)
    for r in range(rows):
        out[r] = np.sort(rng.choice(window, size=k, replace=False))
    return out
