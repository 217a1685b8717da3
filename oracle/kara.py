"""Kara oracle: window scoring, top-k selection, Token2Chunk and paged compaction (fp64, CPU).

TEST INFRASTRUCTURE ONLY (see the package docstring). Plain numpy, no blocking, no fusion.

What the pages fix, and where (page title, then section):

* "Kara: Efficient Reasoning LLM Serving via Sliding-Window KV Cache Compression", English
  abstract: compression runs at decode time on the recently generated context only (a sliding
  window); bidirectional attention scores and selects informative KV pairs in the window; a
  Token2Chunk module expands a subset of the selected pairs into chunks; the method is adapted
  to PagedAttention. Same page, "method details" (key design): bidirectional attention scores
  the KV pairs, Token2Chunk builds chunks from the selected pairs.
* gist.science explainer (German), section 1 "Zwei-Wege-Konversations-Bewertung": a token that
  the current reasoning refers to strongly gets a high score and is kept. Section 2
  "Token2Chunk": the span between two important points is kept as one flexible-length chunk.
  Results section: about 20 % of the notes are kept.

Readings taken where the pages are silent (each one is used identically by the CUDA library):

* Window = cache slots [n-W, n) of a sequence with n = ctx_len >= W.
* Score of window key j for KV head g = sum over the G query heads h of g and over all window
  queries i of softmax_j(q_hi . k_gj * scale), unmasked (bidirectional), scale = 1/sqrt(d).
  Aggregation = sum (the pages do not name one).
* Selection = the k largest scores, ties broken towards the lower index; output ascending.
* Token2Chunk = anchors (the top ``num_anchors`` of the selection), gap fill between consecutive
  anchors whose gap is at most ``gap_limit``, widening of each anchor by ``widen`` on each
  side, then a trim back to exactly k by (priority, score, index); see ``token2chunk``.
* Compaction = deterministic allocation of fresh blocks from a LIFO free list, copy of the
  first window page's prefix rows and of the kept rows, block-table rewrite, free of the old
  window blocks; see ``compact``.
* Variants the pages leave open (``window_scores_agg``, ``shared_keep``, ``trim="chunk"``):
  the mean (the sum over its G * W pairs) and the max (the largest probability any query
  gives the key) in place of the sum; one selection per layer shared by its KV heads
  (selection and Token2Chunk on the head-summed scores); and a chunk-aware trim that drops
  whole unanchored runs of the union, weakest first, before it trims single tokens.

Parity pins (tests/test_oracle_kara.py): closed forms for two keys, a dominant key (catches a
transposed sum), equal keys, GQA group mapping, scale, the W*G total, brute force by pairwise
dominance for selection and trim, hand-worked golden cases, invariants of Token2Chunk and of
compaction (conservation, untouched blocks); for the variants, a brute-force max with its
bounds, closed forms, the mean against the sum, hand-worked golden cases of the shared
selection and of the chunk-aware trim. No function here is unpinned.
"""

from __future__ import annotations

import numpy as np

OK = 0
ERR_INVALID_ARG = 1
ERR_OUT_OF_BLOCKS = 3


# --------------------------------------------------------------------------------------------
# Window scoring
# --------------------------------------------------------------------------------------------

def window_slots(n: int, window: int) -> np.ndarray:
    """Cache slots of the compression window of a sequence holding n tokens: [n-W, n)."""
    if n < window:
        raise ValueError("window longer than the cached context")
    return np.arange(n - window, n)


def gather_rows(pool: np.ndarray, table_row: np.ndarray, slots: np.ndarray, page: int) -> np.ndarray:
    """Rows of a paged pool [num_blocks, page, ...] for the given logical slots of one sequence."""
    blocks = table_row[slots // page]
    return pool[blocks, slots % page]


def window_probs(q_win: np.ndarray, k_win: np.ndarray, scale: float) -> np.ndarray:
    """Bidirectional (unmasked) attention inside the window.

    q_win: [W, Hq, d] float64, k_win: [W, Hkv, d] float64. Returns p[h, i, j] =
    softmax over j of (q_hi . k_{g(h) j}) * scale, with g(h) = h // (Hq // Hkv).
    """
    w, hq, _ = q_win.shape
    hkv = k_win.shape[1]
    group = hq // hkv
    p = np.empty((hq, w, w))
    for h in range(hq):
        g = h // group
        s = (q_win[:, h, :] @ k_win[:, g, :].T) * scale  # [i, j]
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        p[h] = e / e.sum(axis=1, keepdims=True)
    return p


def window_scores(q_win: np.ndarray, k_win: np.ndarray, scale: float) -> np.ndarray:
    """Per-token importance of the window keys, [Hkv, W]: column sums of the softmax over the
    window queries and over the query heads of each GQA group."""
    hq = q_win.shape[1]
    hkv = k_win.shape[1]
    group = hq // hkv
    p = window_probs(q_win, k_win, scale)
    out = np.zeros((hkv, q_win.shape[0]))
    for h in range(hq):
        out[h // group] += p[h].sum(axis=0)
    return out


def window_scores_agg(q_win: np.ndarray, k_win: np.ndarray, scale: float,
                      agg: str) -> np.ndarray:
    """Aggregation variants of the window scores, [Hkv, W] (the pages name no aggregation;
    sum is the main reading, these are the variants it leaves open):
    "sum"  - window_scores;
    "mean" - the sum divided by the G * W (query head, window query) pairs it runs over;
    "max"  - the largest softmax probability any window query of any query head of the group
             gives the key."""
    if agg == "sum":
        return window_scores(q_win, k_win, scale)
    hq = q_win.shape[1]
    hkv = k_win.shape[1]
    group = hq // hkv
    if agg == "mean":
        return window_scores(q_win, k_win, scale) / (group * q_win.shape[0])
    if agg == "max":
        p = window_probs(q_win, k_win, scale)
        out = np.zeros((hkv, q_win.shape[0]))
        for h in range(hq):
            out[h // group] = np.maximum(out[h // group], p[h].max(axis=0))
        return out
    raise ValueError(agg)


def shared_keep(scores: np.ndarray, k: int, num_anchors: int, gap_limit: int,
                widen: int) -> np.ndarray:
    """A selection shared by the KV heads of a layer (a variant the pages leave open): the
    per-head scores [Hkv, W] are summed over the heads, selection and Token2Chunk run once on
    the sum, and every head keeps the same positions. Returns keep [Hkv, k]."""
    total = scores.sum(axis=0)
    keep = token2chunk(total, select_topk(total, k), num_anchors, gap_limit, widen)
    return np.repeat(keep[None, :], scores.shape[0], axis=0)


def score_batch(q_win: np.ndarray, k_pool: np.ndarray, block_table: np.ndarray,
                ctx_len: np.ndarray, seq_ids, window: int, scale: float, page: int) -> np.ndarray:
    """Scores for every due sequence: q_win [R, W, Hq, d] float64 (row r is sequence
    seq_ids[r]), k_pool [num_blocks, page, Hkv, d] float64. Returns [R, Hkv, W]."""
    rows = []
    for r, b in enumerate(seq_ids):
        slots = window_slots(int(ctx_len[b]), window)
        k_win = gather_rows(k_pool, block_table[b], slots, page)
        rows.append(window_scores(q_win[r], k_win, scale))
    return np.stack(rows)


# --------------------------------------------------------------------------------------------
# Selection
# --------------------------------------------------------------------------------------------

def select_topk(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores of one window (ties: lower index first), ascending."""
    w = scores.shape[0]
    order = np.lexsort((np.arange(w), -scores))  # primary: score descending, then index ascending
    return np.sort(order[:k])


def select_batch(scores: np.ndarray, k: int) -> np.ndarray:
    """select_topk over every leading index of scores [..., W] -> [..., k] int32."""
    flat = scores.reshape(-1, scores.shape[-1])
    out = np.stack([select_topk(row, k) for row in flat]) if flat.shape[0] else np.zeros((0, k))
    return out.reshape(scores.shape[:-1] + (k,)).astype(np.int32)


# --------------------------------------------------------------------------------------------
# Token2Chunk
# --------------------------------------------------------------------------------------------

def token2chunk_detail(scores: np.ndarray, sel: np.ndarray, num_anchors: int, gap_limit: int,
                       widen: int, trim: str = "token") -> dict:
    """Token2Chunk on one window, step by step, in window coordinates.

    a. Anchors: the ``num_anchors`` selected positions with the largest scores (ties: lower
       index first).
    b. Gap fill: for consecutive anchors a < b (position order) with 1 <= b-a-1 <= gap_limit,
       every position strictly between them is added.
    c. Widen: every position within ``widen`` of an anchor (clipped to the window) is added.
    d. U = selection | fill | widen.
    e. Priority: 2 for an anchor; 1 for a non-anchor member of U that lies in a maximal run of
       consecutive U positions containing an anchor; 0 otherwise.
    f. Keep: the k members of U with the largest (priority, score, -index), ascending.

    trim="chunk" (the chunk-aware trim, a variant the pages leave open) first drops whole
    runs of U that hold no anchor: weakest first, a run's strength being its best score (ties:
    the later run first), as long as the whole run fits in the excess |U| - k; at the first run
    that does not fit it stops, and the rest of the excess is trimmed as in f.
    """
    w = scores.shape[0]
    k = len(sel)
    sel_scores = scores[sel]
    order = np.lexsort((sel, -sel_scores))
    anchors = np.sort(sel[order[:num_anchors]])

    fill = set()
    for a, b in zip(anchors[:-1], anchors[1:]):
        gap = int(b) - int(a) - 1
        if 1 <= gap <= gap_limit:
            fill.update(range(int(a) + 1, int(b)))

    wide = set()
    for a in anchors:
        for p in range(int(a) - widen, int(a) + widen + 1):
            if 0 <= p < w:
                wide.add(p)

    union = set(int(x) for x in sel) | fill | wide
    in_u = np.zeros(w, dtype=bool)
    in_u[list(union)] = True
    is_anchor = np.zeros(w, dtype=bool)
    is_anchor[anchors] = True

    priority = np.full(w, -1, dtype=np.int64)
    p = 0
    while p < w:
        if not in_u[p]:
            p += 1
            continue
        q = p
        while q < w and in_u[q]:
            q += 1
        run_has_anchor = bool(is_anchor[p:q].any())
        for x in range(p, q):
            priority[x] = 2 if is_anchor[x] else (1 if run_has_anchor else 0)
        p = q

    dropped = set()
    if trim == "chunk":
        runs = []                       # (best score, start, positions) of unanchored runs
        p = 0
        while p < w:
            if not in_u[p]:
                p += 1
                continue
            q = p
            while q < w and in_u[q]:
                q += 1
            if not is_anchor[p:q].any():
                runs.append((float(scores[p:q].max()), p, list(range(p, q))))
            p = q
        excess = len(union) - k
        for best, start, pos in sorted(runs, key=lambda r: (r[0], -r[1])):
            if len(pos) > excess:
                break
            dropped.update(pos)
            excess -= len(pos)
    elif trim != "token":
        raise ValueError(trim)

    members = np.array(sorted(union - dropped), dtype=np.int64)
    order = np.lexsort((members, -scores[members], -priority[members]))
    keep = np.sort(members[order[:k]])
    return {
        "anchors": anchors, "fill": np.array(sorted(fill), dtype=np.int64),
        "widen": np.array(sorted(wide), dtype=np.int64),
        "union": np.array(sorted(union), dtype=np.int64),
        "dropped_runs": np.array(sorted(dropped), dtype=np.int64),
        "priority": priority, "keep": keep,
    }


def token2chunk(scores: np.ndarray, sel: np.ndarray, num_anchors: int, gap_limit: int,
                widen: int, trim: str = "token") -> np.ndarray:
    """Kept window positions after Token2Chunk (exactly len(sel) of them, ascending)."""
    return token2chunk_detail(scores, sel, num_anchors, gap_limit, widen, trim)["keep"]


def token2chunk_batch(scores: np.ndarray, sel: np.ndarray, num_anchors: int, gap_limit: int,
                      widen: int, trim: str = "token") -> np.ndarray:
    """token2chunk over every leading index: scores [..., W], sel [..., k] -> [..., k]."""
    fs = scores.reshape(-1, scores.shape[-1])
    fk = sel.reshape(-1, sel.shape[-1])
    out = [token2chunk(fs[i], fk[i], num_anchors, gap_limit, widen, trim)
           for i in range(fs.shape[0])]
    out = np.stack(out) if out else np.zeros((0, sel.shape[-1]))
    return out.reshape(sel.shape).astype(np.int32)


def anchors_for(anchor_frac: float, k: int) -> int:
    """Number of anchors for an anchor fraction: ceil(anchor_frac * k), clipped to [0, k]. The
    product is rounded to 6 decimals first, so that a fraction given in single precision (0.2
    as 0.2000000030) counts as the decimal it stands for."""
    n = int(np.ceil(np.rint(anchor_frac * k * 1e6) / 1e6))
    return max(0, min(k, n))


# --------------------------------------------------------------------------------------------
# Paged compaction
# --------------------------------------------------------------------------------------------

def compact(k_pools, v_pools, block_table, ctx_len, free_list, free_top: int, seq_ids,
            window: int, keep: np.ndarray, page: int):
    """Compaction of the compressed windows into fresh PagedAttention blocks.

    k_pools / v_pools: one array per layer, [num_blocks, page, Hkv, d] of any dtype (the copy is
    bit-exact). keep: [L, R, Hkv, k] window positions kept per (layer, due sequence, KV head).

    For each due sequence b, in the order of seq_ids: off = (n-W) mod page, p0 = (n-W) // page,
    the window covers n_old = ceil((off+W)/page) pages from p0; the compressed window needs
    n_new = ceil((off+k)/page) fresh pages, popped from the top of the free list (stack[top-1]
    first) and assigned to pages p0, p0+1, ... in order. Every layer and KV head then writes
    slot p0*page + t <- slot p0*page + t for t < off (the first window page's prefix) and slot
    n-W+t <- slot n-W+keep[t] for t < k. The table gets the fresh ids at [p0, p0+n_new) and -1
    at [p0+n_new, p0+n_old); ctx_len becomes n-W+k; once every sequence has popped, the old
    window blocks are pushed (sequence order, page order). If the free list holds fewer blocks
    than the sequences need together, nothing changes and the status is ERR_OUT_OF_BLOCKS.
    Every keep row must list window positions (0 <= keep < W) in strictly ascending order
    (the compressed window keeps the order of the tokens it retains); otherwise nothing
    changes and the status is ERR_INVALID_ARG.

    Returns (status, k_pools, v_pools, block_table, ctx_len, free_list, free_top, fresh_ids),
    all new arrays; fresh_ids maps each due sequence to its fresh block ids.
    """
    kp = [x.copy() for x in k_pools]
    vp = [x.copy() for x in v_pools]
    bt = block_table.copy()
    cl = ctx_len.copy()
    fl = free_list.copy()
    top = int(free_top)
    k = keep.shape[-1]

    rows = keep.reshape(-1, k) if keep.size else keep.reshape(0, max(k, 1))
    for row in rows:
        if (row < 0).any() or (row >= window).any() or (np.diff(row) <= 0).any():
            return (ERR_INVALID_ARG, kp, vp, bt, cl, fl, top, {})

    plans = []
    need = 0
    for b in seq_ids:
        n = int(cl[b])
        if n < window or k > window:
            return (ERR_INVALID_ARG, kp, vp, bt, cl, fl, top, {})
        start = n - window
        off, p0 = start % page, start // page
        n_old = -(-(off + window) // page)
        n_new = -(-(off + k) // page)
        plans.append((b, n, start, off, p0, n_old, n_new))
        need += n_new
    if need > top:
        return (ERR_OUT_OF_BLOCKS, kp, vp, bt, cl, fl, top, {})

    fresh_ids = {}
    for (b, n, start, off, p0, n_old, n_new) in plans:
        ids = [int(fl[top - 1 - i]) for i in range(n_new)]
        top -= n_new
        fresh_ids[int(b)] = ids

    old_tables = {int(b): bt[b].copy() for b in seq_ids}
    for r, (b, n, start, off, p0, n_old, n_new) in enumerate(plans):
        src_table = old_tables[int(b)]
        ids = fresh_ids[int(b)]

        def dst(slot):
            return ids[slot // page - p0], slot % page

        def src(slot):
            return int(src_table[slot // page]), slot % page

        for layer in range(len(kp)):
            for t in range(off):
                slot = p0 * page + t
                db, dr = dst(slot)
                sb, sr = src(slot)
                kp[layer][db, dr] = k_pools[layer][sb, sr]
                vp[layer][db, dr] = v_pools[layer][sb, sr]
            hkv = kp[layer].shape[2]
            for g in range(hkv):
                for t in range(k):
                    sb, sr = src(start + int(keep[layer, r, g, t]))
                    db, dr = dst(start + t)
                    kp[layer][db, dr, g] = k_pools[layer][sb, sr, g]
                    vp[layer][db, dr, g] = v_pools[layer][sb, sr, g]
        for i in range(n_old):
            bt[b, p0 + i] = ids[i] if i < n_new else -1
        cl[b] = start + k

    for (b, n, start, off, p0, n_old, n_new) in plans:
        for i in range(n_old):
            fl[top] = old_tables[int(b)][p0 + i]
            top += 1
    return (OK, kp, vp, bt, cl, fl, top, fresh_ids)
