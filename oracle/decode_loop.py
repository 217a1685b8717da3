"""Decode loop with periodic Kara compression (fp64 where it computes, CPU).

TEST INFRASTRUCTURE ONLY (see the package docstring). Plain numpy, one sequence at a time.

What the pages fix, and where (page title, then section):

* "Kara: Efficient Reasoning LLM Serving via Sliding-Window KV Cache Compression", English
  abstract: compression happens during decoding and looks only at the recently generated
  context; the kept pairs serve the decoding that follows; a threshold-triggered policy is
  what the method avoids.
* gist.science explainer (German), section 3 "Der 'Periodische' Zeitplan (KvLLM)", and the
  Japanese explainer's matching section: instead of waiting until the cache is nearly full,
  KvLLM cleans up on a fixed schedule, every 100 steps, for some selected requests, taking the
  oldest part of the current reasoning.

Readings taken where the pages are silent (each one is used identically by the CUDA library):

* One decode step appends one token per sequence: for every layer, the token's query attends
  over the cached slots [0, n) and over itself (slot n), and its key and value go to slot n.
  The block for slot n is taken when n starts a page (n % page == 0), before any layer runs:
  sequences in ascending order pop from the top of the free list (stack[top-1] first). Then
  ctx_len becomes n + 1.
* tail[b] counts the tokens appended since the sequence was last compressed (the prompt is
  never compressed). Every ``period`` steps (the pages: 100) the sequences with tail >= W are
  due; a due sequence's window is its last W slots [n-W, n), the window that the compression
  calls take, and its tail returns to 0 after the compression. With a check every step the
  window is exactly the uncompressed tail; with a longer period up to period - 1 older
  uncompressed tokens stay where they are.
* LaCache in the same loop ("LaCache: Ladder-Shaped KV Caching ...", iterative compaction:
  the ladder is applied again whenever the cache fills up; experimental setup: a fixed
  budget per layer): at a check step a sequence is also due when its length reaches the
  capacity sink + recent + R_max, the length at which one ladder pass keeps exactly the
  budget in every layer; the pass then runs over its whole cache (lacache.lacache_compact).
* The window queries come from a per-sequence ring of 2W rows per layer: the query of the
  token at slot s is stored at rows s mod W and s mod W + W, so the queries of slots
  [n-W, n) are rows (n-W) mod W .. (n-W) mod W + W - 1, contiguous.

Parity pins (tests/test_oracle_decode_loop.py): a dense model of the same loop (plain Python
lists of K/V rows and queries per sequence, no block table, no ring) gives the same cache
contents through the block table, the same window queries and the same attention outputs
(computed there directly as a softmax); block conservation; the allocation order; nothing
changes when the free list runs short; the trigger fires exactly at check steps for tails of
at least W. No function here is unpinned.
"""

from __future__ import annotations

import numpy as np

from . import decode

OK = 0
ERR_INVALID_ARG = 1
ERR_OUT_OF_BLOCKS = 3


def step_begin(block_table: np.ndarray, ctx_len: np.ndarray, free_list: np.ndarray,
               free_top: int, page: int):
    """Blocks for this step's new slots. Returns (status, block_table, free_top), new arrays;
    on an error nothing changes."""
    bt = block_table.copy()
    top = int(free_top)
    need = [b for b in range(len(ctx_len)) if int(ctx_len[b]) % page == 0]
    for b in need:
        if int(ctx_len[b]) // page >= bt.shape[1]:
            return ERR_INVALID_ARG, block_table.copy(), int(free_top)
    if len(need) > top:
        return ERR_OUT_OF_BLOCKS, block_table.copy(), int(free_top)
    for j, b in enumerate(need):
        bt[b, int(ctx_len[b]) // page] = free_list[top - 1 - j]
    return OK, bt, top - len(need)


def decode_append(q: np.ndarray, k_new: np.ndarray, v_new: np.ndarray, k_pool: np.ndarray,
                  v_pool: np.ndarray, block_table: np.ndarray, ctx_len: np.ndarray,
                  scale: float, page: int, q_ring: np.ndarray | None, window: int):
    """One layer of one decode step. q [B, Hq, d]; k_new, v_new [B, Hkv, d] (the new token);
    k_pool, v_pool [num_blocks, page, Hkv, d]; q_ring [B, 2W, Hq, d] or None.

    Writes the new token's K/V to slot n = ctx_len[b] and its query to ring rows n mod W and
    n mod W + W, then attends over slots [0, n] (decode.decode_attention on ctx_len + 1).
    Returns (out [B, Hq, d] float64, k_pool, v_pool, q_ring), new arrays."""
    kp, vp = k_pool.copy(), v_pool.copy()
    ring = None if q_ring is None else q_ring.copy()
    for b in range(len(ctx_len)):
        n = int(ctx_len[b])
        blk = int(block_table[b, n // page])
        kp[blk, n % page] = k_new[b]
        vp[blk, n % page] = v_new[b]
        if ring is not None:
            ring[b, n % window] = q[b]
            ring[b, n % window + window] = q[b]
    out = decode.decode_attention(q.astype(np.float64), kp.astype(np.float64),
                                  vp.astype(np.float64), block_table, ctx_len + 1, scale, page)
    return out, kp, vp, ring


def step_end(ctx_len: np.ndarray, tail: np.ndarray | None, window: int, check: bool,
             capacity: int = 0):
    """ctx_len + 1, tail + 1, and on a check step the due sequences (ascending): tail >= W
    (when W > 0, Kara) or ctx_len >= capacity (when capacity > 0, LaCache)."""
    cl = ctx_len + 1
    tl = None if tail is None else tail + 1
    due = [b for b in range(len(cl))
           if check and ((window > 0 and tl is not None and int(tl[b]) >= window)
                         or (capacity > 0 and int(cl[b]) >= capacity))]
    return cl, tl, due


def window_queries(q_ring: np.ndarray, ctx_len: np.ndarray, seq_ids, window: int) -> np.ndarray:
    """q_win [R, W, Hq, d] of the due sequences, read from the ring: window position i of
    sequence b is ring row (n - W) mod W + i."""
    out = []
    for b in seq_ids:
        start = (int(ctx_len[b]) - window) % window
        out.append(q_ring[b, start:start + window])
    return np.stack(out)


def reset_tails(tail: np.ndarray, seq_ids) -> np.ndarray:
    tl = tail.copy()
    for b in seq_ids:
        tl[b] = 0
    return tl
