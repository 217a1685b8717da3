"""Pins of the Kara oracle against closed forms, invariants, brute force and golden cases.

Each test would fail under a plausible mistake in the oracle: a dropped term, a wrong sign or
index, a transposed sum, a causal mask, a wrong GQA mapping or scale.
"""

import math
import os

import numpy as np
import pytest

from oracle import kara as ok

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


# ------------------------------------------------------------------ scoring

def test_softmax_rows_sum_to_one():
    q, k = rnd(1, 16, 4, 8), rnd(2, 16, 2, 8)
    p = ok.window_probs(q, k, 1 / math.sqrt(8))
    assert np.allclose(p.sum(axis=2), 1.0, atol=1e-12, rtol=0)
    assert (p >= 0).all()


@pytest.mark.parametrize("w,hq,hkv", [(8, 2, 1), (16, 4, 2), (33, 6, 2), (7, 3, 3)])
def test_scores_total_is_window_times_group(w, hq, hkv):
    q, k = rnd(3, w, hq, 16), rnd(4, w, hkv, 16)
    s = ok.window_scores(q, k, 0.25)
    assert s.shape == (hkv, w)
    assert np.allclose(s.sum(axis=1), w * (hq // hkv), rtol=1e-12)


def test_two_keys_closed_form():
    # W=2, one head: score_0 = sum_i logistic((s_i0 - s_i1)).
    d = 4
    q = np.array([[[1.0, 2.0, 0.0, 0.0]], [[-0.5, 0.25, 3.0, 0.0]]])     # [W=2, 1, d]
    k = np.array([[[0.5, 0.0, 1.0, 0.0]], [[0.0, 1.0, -1.0, 2.0]]])
    scale = 1 / math.sqrt(d)
    s = ok.window_scores(q, k, scale)
    expect0 = 0.0
    for i in range(2):
        a = sum(q[i, 0, t] * k[0, 0, t] for t in range(d)) * scale
        b = sum(q[i, 0, t] * k[1, 0, t] for t in range(d)) * scale
        expect0 += 1.0 / (1.0 + math.exp(b - a))
    assert s[0, 0] == pytest.approx(expect0, rel=1e-13)
    assert s[0, 1] == pytest.approx(2.0 - expect0, rel=1e-13)


def test_scale_enters_as_one_over_sqrt_d():
    # q = e0, k0 = c*e0, k1 = 0  => p_i0 = logistic(c * scale) for both queries.
    for d in (4, 16, 64):
        q = np.zeros((2, 1, d)); q[:, 0, 0] = 1.0
        k = np.zeros((2, 1, d)); k[0, 0, 0] = 3.0
        s = ok.window_scores(q, k, 1 / math.sqrt(d))
        assert s[0, 0] == pytest.approx(2 / (1 + math.exp(-3 / math.sqrt(d))), rel=1e-13)


def test_dominant_last_key_gets_everything():
    # Unmasked: every query (including the first) sees the last key. A causal mask or a row
    # sum instead of a column sum would both fail this.
    w, d = 8, 8
    q = np.ones((w, 2, d))
    k = np.zeros((w, 1, d)); k[-1, 0, :] = 20.0
    s = ok.window_scores(q, k, 1 / math.sqrt(d))
    assert s[0, -1] == pytest.approx(w * 2, rel=1e-9)
    assert s[0, :-1].max() < 1e-9


def test_equal_keys_give_group_size():
    w, d = 12, 8
    q = rnd(5, w, 6, d)
    k = np.tile(rnd(6, 1, 2, d), (w, 1, 1))
    s = ok.window_scores(q, k, 1 / math.sqrt(d))
    assert np.allclose(s, 3.0, rtol=1e-12)


def test_gqa_group_mapping():
    # Hq=4, Hkv=2: heads 0,1 read KV head 0; heads 2,3 read KV head 1 (h // G, not h % Hkv).
    w, d = 8, 4
    q = np.zeros((w, 4, d)); q[:, :, 0] = 1.0
    k = np.zeros((w, 2, d))
    k[1, 0, 0] = 80.0      # KV head 0: key 1 dominates
    k[5, 1, 0] = 80.0      # KV head 1: key 5 dominates
    s = ok.window_scores(q, k, 0.5)
    assert s[0, 1] == pytest.approx(2 * w, rel=1e-6)
    assert s[1, 5] == pytest.approx(2 * w, rel=1e-6)


def test_brute_force_tiny_windows():
    # Scalar loops without the max shift (values are small enough not to overflow).
    rng = np.random.default_rng(7)
    for w in (1, 2, 3, 5, 8):
        hq, hkv, d = 4, 2, 3
        q, k = rng.standard_normal((w, hq, d)), rng.standard_normal((w, hkv, d))
        s = ok.window_scores(q, k, 0.7)
        for g in range(hkv):
            for j in range(w):
                tot = 0.0
                for h in range(g * 2, g * 2 + 2):
                    for i in range(w):
                        num = math.exp(0.7 * sum(q[i, h, t] * k[j, g, t] for t in range(d)))
                        den = sum(math.exp(0.7 * sum(q[i, h, t] * k[jj, g, t] for t in range(d)))
                                  for jj in range(w))
                        tot += num / den
                assert s[g, j] == pytest.approx(tot, rel=1e-12)


def test_large_logits_are_stable():
    q, k = 1000 * rnd(8, 16, 2, 8), rnd(9, 16, 1, 8)
    s = ok.window_scores(q, k, 1.0)
    assert np.isfinite(s).all()
    assert s.sum() == pytest.approx(32.0, rel=1e-12)


def test_paged_window_gather_reads_the_last_w_slots():
    page, n, w = 4, 11, 6
    pool = np.arange(5 * page).reshape(5, page, 1, 1).astype(float)
    table = np.array([3, 0, 4, 1])
    got = ok.gather_rows(pool, table, ok.window_slots(n, w), page)[:, 0, 0]
    # slots 5..10 -> (page 1, rows 1..3) -> block 0 rows 1..3, (page 2, rows 0..2) -> block 4
    assert got.tolist() == [1, 2, 3, 16, 17, 18]


# ------------------------------------------------------------------ selection

def dominance_select(s, k):
    w = len(s)
    out = []
    for j in range(w):
        beaten_by = sum(1 for i in range(w) if s[i] > s[j] or (s[i] == s[j] and i < j))
        if beaten_by < k:
            out.append(j)
    return out


@pytest.mark.parametrize("seed", range(20))
def test_select_matches_dominance_brute_force(seed):
    rng = np.random.default_rng(seed)
    w = int(rng.integers(1, 14))
    k = int(rng.integers(1, w + 1))
    s = rng.integers(0, 4, size=w).astype(float)       # many ties
    assert ok.select_topk(s, k).tolist() == dominance_select(s, k)


def test_select_invariants_and_ties():
    s = np.array([1.0, 3.0, 3.0, 0.5, 3.0, 2.0])
    sel = ok.select_topk(s, 2)
    assert sel.tolist() == [1, 2]                       # ties go to the lower index
    rng = np.random.default_rng(11)
    s = rng.random(1024)
    sel = ok.select_topk(s, 204)
    assert len(sel) == 204 and np.all(np.diff(sel) > 0)
    rest = np.setdiff1d(np.arange(1024), sel)
    assert s[sel].min() >= s[rest].max()
    assert ok.select_topk(s[:16], 16).tolist() == list(range(16))


# ------------------------------------------------------------------ Token2Chunk

def load_golden(name):
    cases = []
    cur = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if line == "---":
                if cur:
                    cases.append(cur)
                cur = {}
                continue
            key, val = line.split(":", 1)
            cur[key.strip()] = [float(x) for x in val.split()] if val.strip() else []
    if cur:
        cases.append(cur)
    return cases


def test_token2chunk_golden_cases():
    cases = load_golden("token2chunk_cases.txt")
    assert len(cases) >= 3
    for c in cases:
        scores = np.array(c["scores"])
        sel = np.array(c["sel"], dtype=np.int64)
        det = ok.token2chunk_detail(scores, sel, int(c["num_anchors"][0]), int(c["gap_limit"][0]),
                                    int(c["widen"][0]))
        assert det["anchors"].tolist() == [int(x) for x in c["anchors"]]
        assert det["union"].tolist() == [int(x) for x in c["union"]]
        assert det["keep"].tolist() == [int(x) for x in c["keep"]]


def test_chunk_trim_golden_cases():
    # hand-worked cases (tests/golden/chunk_trim_cases.txt): whole unanchored runs dropped
    # weakest first while they fit, the stop rule, equal strengths, several runs
    cases = load_golden("chunk_trim_cases.txt")
    assert len(cases) >= 4
    for c in cases:
        scores = np.array(c["scores"])
        sel = np.array(c["sel"], dtype=np.int64)
        args = (scores, sel, int(c["num_anchors"][0]), int(c["gap_limit"][0]), int(c["widen"][0]))
        det = ok.token2chunk_detail(*args, trim="chunk")
        assert det["union"].tolist() == [int(x) for x in c["union"]]
        assert det["dropped_runs"].tolist() == [int(x) for x in c["dropped_runs"]]
        assert det["keep"].tolist() == [int(x) for x in c["keep"]]
        assert ok.token2chunk(*args).tolist() == [int(x) for x in c["keep_token"]]


@pytest.mark.parametrize("seed", range(40))
def test_chunk_trim_invariants(seed):
    # |keep| = k, anchors kept, keep within U, every run dropped whole is an unanchored run of
    # U, and no kept token of an unanchored run is weaker than a dropped run's best token
    # unless the trim fell back to tokens; with no excess both trims keep U
    scores, sel, na, gap, wid = t2c_random_case(seed)
    k = len(sel)
    det = ok.token2chunk_detail(scores, sel, na, gap, wid, trim="chunk")
    keep = set(det["keep"].tolist())
    union = set(det["union"].tolist())
    assert len(keep) == k and set(det["anchors"].tolist()) <= keep <= union
    dropped = set(det["dropped_runs"].tolist())
    assert not (dropped & keep) and not (dropped & set(det["anchors"].tolist()))
    assert len(union) - len(dropped) >= k
    for p in dropped:                       # dropped positions form whole runs of U
        for q in (p - 1, p + 1):
            if q in union:
                assert q in dropped
    if len(union) == k:
        assert keep == union
    if not dropped:
        assert det["keep"].tolist() == ok.token2chunk(scores, sel, na, gap, wid).tolist()


def t2c_random_case(seed):
    rng = np.random.default_rng(seed)
    w = int(rng.integers(4, 40))
    k = int(rng.integers(1, w + 1))
    scores = rng.integers(0, 6, size=w).astype(float) + rng.random(w) * (seed % 2)
    sel = ok.select_topk(scores, k)
    na = int(rng.integers(0, k + 1))
    gap = int(rng.integers(0, 6))
    wid = int(rng.integers(0, 3))
    return scores, sel, na, gap, wid


@pytest.mark.parametrize("seed", range(40))
def test_token2chunk_invariants(seed):
    scores, sel, na, gap, wid = t2c_random_case(seed)
    w, k = len(scores), len(sel)
    det = ok.token2chunk_detail(scores, sel, na, gap, wid)
    keep, anchors, union = det["keep"], det["anchors"], det["union"]
    assert len(keep) == k and np.all(np.diff(keep) > 0)
    assert set(anchors.tolist()) <= set(keep.tolist()) <= set(union.tolist())
    assert set(sel.tolist()) <= set(union.tolist())
    # anchors are the top-na of the selection by (score desc, index asc)
    assert anchors.tolist() == sorted(dominance_select_subset(scores, sel, na))
    # fill: exactly the interiors of consecutive-anchor gaps of length 1..gap
    expect_fill = set()
    for a, b in zip(anchors[:-1], anchors[1:]):
        if 0 < b - a - 1 <= gap:
            expect_fill |= set(range(a + 1, b))
    assert set(det["fill"].tolist()) == expect_fill
    for a, b in zip(anchors[:-1], anchors[1:]):
        if b - a - 1 > gap:
            inner = set(range(a + 1, b))
            assert not (inner & set(det["fill"].tolist()))
    # widen: the clipped +-wid neighbourhoods
    expect_w = set()
    for a in anchors:
        expect_w |= set(p for p in range(a - wid, a + wid + 1) if 0 <= p < w)
    assert set(det["widen"].tolist()) == expect_w
    # trim: keep = the k members of U that no more than k-1 others dominate
    pr = det["priority"]
    key = {p: (pr[p], scores[p], -p) for p in union.tolist()}
    expect_keep = [p for p in union.tolist()
                   if sum(1 for o in union.tolist() if key[o] > key[p]) < k]
    assert keep.tolist() == sorted(expect_keep)


def dominance_select_subset(scores, sel, n):
    out = []
    for j in sel:
        beaten = sum(1 for i in sel if scores[i] > scores[j] or (scores[i] == scores[j] and i < j))
        if beaten < n:
            out.append(int(j))
    return out


@pytest.mark.parametrize("seed", range(10))
def test_token2chunk_identity_cases(seed):
    scores, sel, na, gap, wid = t2c_random_case(seed)
    assert ok.token2chunk(scores, sel, 0, gap, wid).tolist() == sel.tolist()
    assert ok.token2chunk(scores, sel, na, 0, 0).tolist() == sel.tolist()


def test_token2chunk_priority_runs():
    # Two anchors 2 and 5 (gap 2 <= 3): run 1..6 has priority 1/2; 9 is an isolated pick.
    scores = np.array([0, 1, 9, 0, 0, 8, 1, 0, 0, 5, 0, 0], dtype=float)
    sel = np.array([2, 5, 9])
    det = ok.token2chunk_detail(scores, sel, 2, 3, 1)
    pr = det["priority"]
    assert pr[2] == 2 and pr[5] == 2
    assert all(pr[p] == 1 for p in (1, 3, 4, 6))
    assert pr[9] == 0
    # 9 (priority 0) is dropped first; among priority 1, scores tie at 1 for slots 1 and 6 and
    # the lower index wins.
    assert det["keep"].tolist() == [1, 2, 5]


def test_anchor_count():
    assert ok.anchors_for(0.5, 204) == 102
    assert ok.anchors_for(0.5, 409) == 205
    assert ok.anchors_for(0.0, 32) == 0
    assert ok.anchors_for(1.0, 32) == 32
    assert ok.anchors_for(0.1, 30) == 3
    assert ok.anchors_for(0.5, 61) == 31                      # ceil(30.5)
    # a fraction that arrives in single precision counts as its decimal: 0.2 as 0.2000000030
    # gives ceil(0.2 * 5) = 1, not 2 (the product is rounded to 6 decimals before the ceiling)
    assert ok.anchors_for(float(np.float32(0.2)), 5) == 1
    assert ok.anchors_for(float(np.float32(0.2)), 61) == 13


# ------------------------------------------------------------------ compaction

def small_pool(seed, page=4, nb=12, hkv=2, d=3, layers=2):
    rng = np.random.default_rng(seed)
    ks = [rng.integers(0, 60000, size=(nb, page, hkv, d)).astype(np.uint16) for _ in range(layers)]
    vs = [rng.integers(0, 60000, size=(nb, page, hkv, d)).astype(np.uint16) for _ in range(layers)]
    return ks, vs


def test_compact_golden_hand_worked():
    # page 4; one sequence of n=11 slots on blocks [7, 2, 5]; window W=6 -> slots 5..10,
    # off = 1, p0 = 1, old pages 1..2 (blocks 2, 5), fresh pages ceil((1+2)/4) = 1.
    # free list [9, 3, 8], top 3 -> block 8 is popped; keep = [1, 4] -> slots 6 and 9.
    page = 4
    ks, vs = small_pool(0, page=page, nb=10, hkv=2, d=3, layers=1)
    table = np.array([[7, 2, 5, -1]], dtype=np.int32)
    ctx = np.array([11], dtype=np.int32)
    free = np.array([9, 3, 8, 0, 0, 0, 0, 0, 0, 0], dtype=np.int32)
    keep = np.array([[[[1, 4], [0, 5]]]], dtype=np.int32)     # [L=1, R=1, Hkv=2, k=2]
    st, kp, vp, bt, cl, fl, top, fresh = ok.compact(ks, vs, table, ctx, free, 3, [0], 6, keep, page)
    assert st == ok.OK
    assert fresh == {0: [8]}
    assert bt.tolist() == [[7, 8, -1, -1]]
    assert cl.tolist() == [7]
    assert top == 4 and fl[:4].tolist() == [9, 3, 2, 5]
    # slot 4 (block 2 row 0) -> block 8 row 0 (prefix, both heads)
    assert (kp[0][8, 0] == ks[0][2, 0]).all()
    # head 0: slot 5 <- slot 6 (block 2 row 2), slot 6 <- slot 9 (block 5 row 1)
    assert (kp[0][8, 1, 0] == ks[0][2, 2, 0]).all() and (kp[0][8, 2, 0] == ks[0][5, 1, 0]).all()
    # head 1: slot 5 <- slot 5 (block 2 row 1), slot 6 <- slot 10 (block 5 row 2)
    assert (vp[0][8, 1, 1] == vs[0][2, 1, 1]).all() and (vp[0][8, 2, 1] == vs[0][5, 2, 1]).all()


def logical(pool, table_row, n, page):
    slots = np.arange(n)
    return pool[table_row[slots // page], slots % page]


@pytest.mark.parametrize("seed", range(8))
def test_compact_logical_view_and_conservation(seed):
    rng = np.random.default_rng(100 + seed)
    page, hkv, d, layers, w = 4, 2, 3, 2, 9
    bsz = 3
    ctx = rng.integers(w, 30, size=bsz).astype(np.int32)
    pages = [-(-int(n) // page) for n in ctx]
    nb = sum(pages) + 12
    perm = rng.permutation(nb)
    table = np.full((bsz, 10), -1, dtype=np.int32)
    pos = 0
    for b in range(bsz):
        table[b, :pages[b]] = perm[pos:pos + pages[b]]
        pos += pages[b]
    free = np.zeros(nb, dtype=np.int32)
    free[:nb - pos] = perm[pos:]
    top = nb - pos
    ks, vs = small_pool(seed, page, nb, hkv, d, layers)
    seq_ids = sorted(rng.choice(bsz, size=2, replace=False).tolist())
    k = int(rng.integers(1, w + 1))
    keep = np.stack([np.stack([np.stack([np.sort(rng.choice(w, k, replace=False))
                                         for _ in range(hkv)]) for _ in seq_ids])
                     for _ in range(layers)]).astype(np.int32)
    st, kp, vp, bt, cl, fl, top2, fresh = ok.compact(ks, vs, table, ctx, free, top, seq_ids, w,
                                                     keep, page)
    assert st == ok.OK
    used = set(int(x) for x in bt.ravel() if x >= 0)
    free_set = set(int(x) for x in fl[:top2])
    assert not (used & free_set) and len(used) + len(free_set) == nb
    touched = set(x for ids in fresh.values() for x in ids)
    for layer in range(layers):
        for blk in range(nb):
            if blk not in touched:
                assert (kp[layer][blk] == ks[layer][blk]).all()
        for r, b in enumerate(seq_ids):
            n = int(ctx[b])
            assert cl[b] == n - w + k
            new = logical(kp[layer], bt[b], n - w + k, page)
            old = logical(ks[layer], table[b], n, page)
            assert (new[:n - w] == old[:n - w]).all()
            for g in range(hkv):
                assert (new[n - w:, g] == old[n - w + keep[layer, r, g], g]).all()
        for b in set(range(bsz)) - set(seq_ids):
            assert (bt[b] == table[b]).all() and cl[b] == ctx[b]


def test_compact_out_of_blocks_changes_nothing():
    page = 4
    ks, vs = small_pool(3, page=page, nb=6, hkv=1, d=2, layers=1)
    table = np.array([[0, 1, 2, 3, -1]], dtype=np.int32)
    ctx = np.array([16], dtype=np.int32)
    free = np.array([4, 5, 0, 0, 0, 0], dtype=np.int32)
    keep = np.arange(12, dtype=np.int32).reshape(1, 1, 1, 12)
    st, kp, vp, bt, cl, fl, top, _ = ok.compact(ks, vs, table, ctx, free, 0, [0], 12, keep, page)
    assert st == ok.ERR_OUT_OF_BLOCKS
    assert (bt == table).all() and (cl == ctx).all() and top == 0


@pytest.mark.parametrize("bad", ["below", "past_window", "repeat", "descending"])
def test_compact_bad_keep_changes_nothing(bad):
    page = 4
    ks, vs = small_pool(5, page=page, nb=10, hkv=2, d=2, layers=2)
    table = np.array([[0, 1, 2, 3, -1]], dtype=np.int32)
    ctx = np.array([16], dtype=np.int32)
    free = np.array([4, 5, 6, 7, 8, 9, 0, 0, 0, 0], dtype=np.int32)
    keep = np.tile(np.arange(0, 12, 2, dtype=np.int32), (2, 1, 2, 1))   # W = 12, k = 6
    st, *_ = ok.compact(ks, vs, table, ctx, free, 6, [0], 12, keep, page)
    assert st == ok.OK
    keep = keep.copy()
    if bad == "below":
        keep[1, 0, 1, 0] = -1
    elif bad == "past_window":
        keep[0, 0, 1, 5] = 12
    elif bad == "repeat":
        keep[1, 0, 0, 3] = keep[1, 0, 0, 2]
    else:
        keep[0, 0, 0, 2], keep[0, 0, 0, 3] = keep[0, 0, 0, 3], keep[0, 0, 0, 2]
    st, kp, vp, bt, cl, fl, top, fresh = ok.compact(ks, vs, table, ctx, free, 6, [0], 12, keep,
                                                    page)
    assert st == ok.ERR_INVALID_ARG and fresh == {}
    assert (bt == table).all() and (cl == ctx).all() and top == 6 and (fl == free).all()
    for layer in range(2):
        assert (kp[layer] == ks[layer]).all() and (vp[layer] == vs[layer]).all()


# ---- aggregation variants and the shared selection (variants the pages leave open) ----

def _rand_window(seed, w=9, hq=4, hkv=2, d=8):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((w, hq, d)), rng.standard_normal((w, hkv, d))


def test_mean_is_the_sum_over_its_pairs():
    q, k = _rand_window(1)
    s = ok.window_scores(q, k, 0.5)
    m = ok.window_scores_agg(q, k, 0.5, "mean")
    assert np.allclose(m * (2 * 9), s, rtol=1e-13)
    assert np.allclose(m.sum(axis=1), 1.0, rtol=1e-12)     # the mean of softmax rows sums to 1


def test_max_brute_force_and_bounds():
    q, k = _rand_window(2, w=6, hq=4, hkv=2, d=5)
    mx = ok.window_scores_agg(q, k, 0.7, "max")
    for g in range(2):
        for j in range(6):
            best = 0.0
            for h in (2 * g, 2 * g + 1):
                for i in range(6):
                    logits = [float(q[i, h] @ k[jj, g]) * 0.7 for jj in range(6)]
                    top = max(logits)
                    den = sum(math.exp(x - top) for x in logits)
                    best = max(best, math.exp(logits[j] - top) / den)
            assert abs(mx[g, j] - best) < 1e-13
    s = ok.window_scores(q, k, 0.7)
    assert np.all(mx <= s + 1e-15) and np.all(mx >= s / (2 * 6) - 1e-15)


def test_max_closed_forms():
    # equal keys: every probability is 1/W
    q = np.random.default_rng(3).standard_normal((5, 2, 4))
    k = np.ones((5, 1, 4))
    assert np.allclose(ok.window_scores_agg(q, k, 1.0, "max"), 1 / 5)
    # two keys, one query, one head: max = the logistic probabilities themselves
    q = np.array([[[1.0, 0.0]], [[0.0, 0.0]]])
    k = np.array([[[2.0, 0.0]], [[0.0, 0.0]]])
    p0 = 1 / (1 + math.exp(-2.0))
    mx = ok.window_scores_agg(q, k, 1.0, "max")
    assert np.allclose(mx[0], [p0, 0.5])      # query 1 has equal logits: 0.5 for both keys


def test_shared_keep_golden_cases():
    # hand-worked cases (tests/golden/shared_keep_cases.txt) in which the shared keep set is
    # neither a per-head selection, nor the selection of the maximum over heads
    cases = load_golden("shared_keep_cases.txt")
    assert len(cases) >= 3
    for c in cases:
        heads = sorted(key for key in c if key.startswith("h"))
        sc = np.array([c[h] for h in heads])
        k, na = int(c["k"][0]), int(c["num_anchors"][0])
        gap, wid = int(c["gap_limit"][0]), int(c["widen"][0])
        keep = ok.shared_keep(sc, k, na, gap, wid)
        expect = [int(x) for x in c["keep"]]
        assert keep.shape == (len(heads), k)
        assert all(row.tolist() == expect for row in keep)
        assert sc.sum(axis=0).tolist() == c["sum"]
        assert ok.select_topk(sc.sum(axis=0), k).tolist() == [int(x) for x in c["sel"]]
        for h in range(len(heads)):
            assert ok.token2chunk(sc[h], ok.select_topk(sc[h], k), na, gap, wid).tolist() != expect
        mx = sc.max(axis=0)
        assert ok.token2chunk(mx, ok.select_topk(mx, k), na, gap, wid).tolist() != expect


def test_shared_keep_is_the_selection_of_the_head_sum():
    rng = np.random.default_rng(4)
    sc = rng.random((3, 40))
    keep = ok.shared_keep(sc, 8, 4, 8, 1)
    total = sc.sum(axis=0)
    ref = ok.token2chunk(total, ok.select_topk(total, 8), 4, 8, 1)
    assert keep.shape == (3, 8) and all(np.array_equal(row, ref) for row in keep)
    one = sc[:1]                               # one KV head: the per-head selection itself
    assert np.array_equal(ok.shared_keep(one, 8, 4, 8, 1)[0],
                          ok.token2chunk(one[0], ok.select_topk(one[0], 8), 4, 8, 1))
