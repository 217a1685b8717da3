"""Paged GQA decode-attention oracle (fp64, CPU).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "Kara: Efficient Reasoning LLM Serving via Sliding-Window KV Cache Compression",
English abstract: the compressed cache keeps the useful KV pairs for subsequent decoding, and
the method is adapted to PagedAttention. The decode step that reads the compressed cache is the
ordinary attention of one new query token per sequence over the cached slots, read through the
block table; for grouped-query attention, query head h reads KV head h // (Hq // Hkv).

Reading: slots [0, ctx_len) of the sequence are attended, unmasked; an empty context gives a
zero output.

Parity pins (tests/test_oracle_decode.py): a one-slot context returns that V row; equal scores
return the mean of V; the result equals torch's softmax(q K^T * scale) V in fp64 on a contiguous
copy of the cache (a library routine of the same definition).
"""

from __future__ import annotations

import numpy as np


def decode_attention(q: np.ndarray, k_pool: np.ndarray, v_pool: np.ndarray,
                     block_table: np.ndarray, ctx_len: np.ndarray, scale: float,
                     page: int) -> np.ndarray:
    """q: [B, Hq, d] float64; k_pool, v_pool: [num_blocks, page, Hkv, d] float64.
    Returns out [B, Hq, d] float64."""
    nb, hq, d = q.shape
    hkv = k_pool.shape[2]
    group = hq // hkv
    out = np.zeros((nb, hq, d))
    for b in range(nb):
        n = int(ctx_len[b])
        if n == 0:
            continue
        slots = np.arange(n)
        blocks = block_table[b][slots // page]
        k = k_pool[blocks, slots % page]  # [n, Hkv, d]
        v = v_pool[blocks, slots % page]
        for h in range(hq):
            g = h // group
            s = (k[:, g, :] @ q[b, h]) * scale
            s = s - s.max()
            e = np.exp(s)
            out[b, h] = (e / e.sum()) @ v[:, g, :]
    return out
