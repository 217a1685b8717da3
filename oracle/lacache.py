"""LaCache ladder-pattern oracle: keep map and iterative ladder compaction (CPU).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "LaCache: Ladder-Shaped KV Caching for Efficient Long-Context Modeling of Large Language
Models" (papercache.org summary):

* "how it works" and "method details / ladder pattern": shallow layers keep earlier tokens,
  deeper layers later ones; states outside the ladder are dropped and the rest packed into a
  smaller 2-D cache; the repeating, expanding pattern spreads coverage as evenly as possible
  over the layers.
* "implementation details and key hyper-parameters": span S = number of consecutive layers
  that keep the same token; overlap O.
* "supplementary details": S about L times the keep ratio (L/4 for language modelling); O =
  S/2 for language modelling.
* "iterative compaction": when the cache is full the ladder is applied again to the already
  compacted cache, so older tokens are compressed more and the freed space goes to new tokens;
  early KV states are dropped first.
* "experimental setup": the first 128 tokens (system prompt) kept untouched on LongBench.

Readings (the pages give no formula):

* O is a number of layers (O = S/2 only reads as a layer count); the garbled gloss "tokens
  kept per layer" is not used. Stride D = S - O; D must divide S and L.
* The ladder acts on cache slots (so it re-applies to a compacted cache). The first ``sink``
  slots and the last ``recent`` slots are kept in every layer. The slots between them (the
  region) are cut into rungs of ``rung`` slots; rung j is kept in the S layers
  (j*D + t) mod L, t = 0..S-1. Every layer then keeps S/L of the region.
* Capacity: the region holds at most R_max = (budget - sink - recent) * L / S slots; the
  oldest region slots beyond R_max are dropped in every layer. Compaction runs only on a full
  cache (region >= R_max) and R_max must be a whole number of ladder periods (rung * L / D
  slots), so every layer keeps exactly ``budget`` slots.
* The compacted sequence is written into ceil(budget/page) fresh blocks popped from the free
  list (stack top first, in sequence order), and all ceil(n/page) old blocks are pushed back
  afterwards, in sequence then page order.

Parity pins (tests/test_oracle_lacache.py): every rung is kept in exactly S cyclically
consecutive layers; adjacent rungs share exactly O layers; every layer keeps exactly the
budget; S = L keeps everything; a hand-enumerated golden ladder for L=4, S=2, O=1; iteration
drops the oldest first; bit-exact copies and block conservation.
"""

from __future__ import annotations

import numpy as np

OK = 0
ERR_INVALID_ARG = 1
ERR_OUT_OF_BLOCKS = 3


def check_params(num_layers: int, span: int, overlap: int, rung: int, budget: int, sink: int,
                 recent: int) -> bool:
    """True when the ladder parameters satisfy the readings above."""
    if not (1 <= span <= num_layers and 0 <= overlap < span and rung >= 1):
        return False
    stride = span - overlap
    if span % stride or num_layers % stride:
        return False
    region_budget = budget - sink - recent
    if sink < 0 or recent < 0 or region_budget <= 0:
        return False
    per_period = rung * span // stride  # region slots one layer keeps per ladder period
    return region_budget % per_period == 0


def region_capacity(num_layers: int, span: int, budget: int, sink: int, recent: int) -> int:
    """R_max: the longest region whose ladder keeps budget - sink - recent slots per layer."""
    return (budget - sink - recent) * num_layers // span


def rung_layers(j: int, num_layers: int, span: int, overlap: int) -> list:
    """Layers that keep rung j: S cyclically consecutive layers starting at j*(S-O)."""
    stride = span - overlap
    return [(j * stride + t) % num_layers for t in range(span)]


def ladder_keep_slots(n: int, num_layers: int, span: int, overlap: int, rung: int, budget: int,
                      sink: int = 0, recent: int = 0) -> list:
    """Kept cache slots of every layer (ascending), for a sequence holding n slots."""
    r_max = region_capacity(num_layers, span, budget, sink, recent)
    if n - sink - recent < r_max:
        raise ValueError("ladder compaction needs a full cache")
    region_start = n - recent - r_max
    keep = [list(range(sink)) for _ in range(num_layers)]
    num_rungs = -(-r_max // rung)
    for j in range(num_rungs):
        lo = region_start + j * rung
        hi = min(lo + rung, n - recent)
        for layer in rung_layers(j, num_layers, span, overlap):
            keep[layer].extend(range(lo, hi))
    for layer in range(num_layers):
        keep[layer].extend(range(n - recent, n))
        keep[layer] = np.array(sorted(keep[layer]), dtype=np.int64)
    return keep


def lacache_compact(k_pools, v_pools, block_table, ctx_len, free_list, free_top: int, seq_ids,
                    span: int, overlap: int, rung: int, budget: int, sink: int, recent: int,
                    page: int):
    """Ladder compaction of the whole cache of every due sequence (one pass).

    Layer l of sequence b keeps the slots ladder_keep_slots(n_b, ...)[l]; the t-th kept slot
    goes to slot t of the compacted sequence (every KV head of the layer alike). Returns
    (status, k_pools, v_pools, block_table, ctx_len, free_list, free_top), all new arrays.
    """
    num_layers = len(k_pools)
    kp = [x.copy() for x in k_pools]
    vp = [x.copy() for x in v_pools]
    bt = block_table.copy()
    cl = ctx_len.copy()
    fl = free_list.copy()
    top = int(free_top)
    if not check_params(num_layers, span, overlap, rung, budget, sink, recent):
        return (ERR_INVALID_ARG, kp, vp, bt, cl, fl, top)
    r_max = region_capacity(num_layers, span, budget, sink, recent)

    need = 0
    for b in seq_ids:
        if int(cl[b]) - sink - recent < r_max:
            return (ERR_INVALID_ARG, kp, vp, bt, cl, fl, top)
        need += -(-budget // page)
    if need > top:
        return (ERR_OUT_OF_BLOCKS, kp, vp, bt, cl, fl, top)

    n_new = -(-budget // page)
    fresh = {}
    for b in seq_ids:
        fresh[int(b)] = [int(fl[top - 1 - i]) for i in range(n_new)]
        top -= n_new

    old_tables = {int(b): bt[b].copy() for b in seq_ids}
    old_len = {int(b): int(cl[b]) for b in seq_ids}
    for b in seq_ids:
        n = old_len[int(b)]
        keep = ladder_keep_slots(n, num_layers, span, overlap, rung, budget, sink, recent)
        ids = fresh[int(b)]
        src_table = old_tables[int(b)]
        for layer in range(num_layers):
            src = keep[layer]
            sb = src_table[src // page]
            sr = src % page
            t = np.arange(budget)
            db = np.array(ids)[t // page]
            dr = t % page
            kp[layer][db, dr] = k_pools[layer][sb, sr]
            vp[layer][db, dr] = v_pools[layer][sb, sr]
        n_old = -(-n // page)
        for p in range(n_old):
            bt[b, p] = ids[p] if p < n_new else -1
        cl[b] = budget

    for b in seq_ids:
        n_old = -(-old_len[int(b)] // page)
        for p in range(n_old):
            fl[top] = old_tables[int(b)][p]
            top += 1
    return (OK, kp, vp, bt, cl, fl, top)
