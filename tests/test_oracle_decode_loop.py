"""Pins of the decode-loop oracle (CPU): a dense model of the same loop, allocation rules, the
trigger. The dense model keeps plain per-sequence lists of K/V rows and queries (no block
table, no free list, no ring) and computes attention directly as a softmax, so a wrong slot, a
wrong block, a wrong ring row or a wrong window shows up as a mismatch."""

import math

import numpy as np
import pytest

from decode_kv_cache_kara_b200 import synth
from oracle import decode_loop as dl
from oracle import kara as ok
from oracle import lacache as ol

LOOP = synth.Workload("loop", batch=3, layers=2, hq=4, hkv=2, head_dim=16, ctx_lo=20, ctx_hi=37,
                      window=16, keep=5, heavy_frac=0.0, spare_blocks=4)


def np32(t):
    return t.float().numpy()


def dense_attention(q, rows_k, rows_v, scale):
    """q [d]; rows_k, rows_v: lists of [d] rows. softmax(q . k * scale) v, directly."""
    k = np.array(rows_k, dtype=np.float64)
    v = np.array(rows_v, dtype=np.float64)
    s = k @ q.astype(np.float64) * scale
    p = np.exp(s - s.max())
    return (p / p.sum()) @ v


def paged_row(pool, bt, b, slot, g, page):
    return pool[int(bt[b, slot // page]), slot % page, g]


def run_loop(wl, seed, steps, period, check_every_step=True):
    cache = synth.make_cache(wl, seed, "cpu", with_queries=False, extra_pages=8)
    page, W, L, G = wl.page, wl.window, wl.layers, wl.group
    scale = 1 / math.sqrt(wl.head_dim)
    kp = [np32(t) for t in cache["k"]]
    vp = [np32(t) for t in cache["v"]]
    bt = cache["block_table"].numpy().astype(np.int64)
    cl = cache["ctx_len"].numpy().astype(np.int64)
    fl = cache["free_list"].numpy().astype(np.int64)
    top = int(cache["free_top"][0])
    tail = np.zeros(wl.batch, dtype=np.int64)
    rings = [np.zeros((wl.batch, 2 * W, wl.hq, wl.head_dim), dtype=np.float32) for _ in range(L)]
    # dense model: rows per (layer, sequence, KV head), queries per (layer, sequence)
    dk = [[[[kp[l][bt[b, s // page], s % page, g] for s in range(cl[b])] for g in range(wl.hkv)]
           for b in range(wl.batch)] for l in range(L)]
    dv = [[[[vp[l][bt[b, s // page], s % page, g] for s in range(cl[b])] for g in range(wl.hkv)]
           for b in range(wl.batch)] for l in range(L)]
    dq = [[[] for _ in range(wl.batch)] for _ in range(L)]
    compressions = 0
    for t in range(steps):
        st, bt, top = dl.step_begin(bt, cl, fl, top, page)
        assert st == dl.OK
        for l in range(L):
            inp = synth.decode_step_inputs(wl, seed, t)[l]
            q, kn, vn = np32(inp["q"]), np32(inp["k"]), np32(inp["v"])
            out, kp[l], vp[l], rings[l] = dl.decode_append(q, kn, vn, kp[l], vp[l], bt, cl, scale,
                                                          page, rings[l], W)
            for b in range(wl.batch):
                dq[l][b].append(q[b])
                for g in range(wl.hkv):
                    dk[l][b][g].append(kn[b, g])
                    dv[l][b][g].append(vn[b, g])
                for h in range(wl.hq):
                    ref = dense_attention(q[b, h], dk[l][b][h // G], dv[l][b][h // G], scale)
                    assert np.allclose(out[b, h], ref, rtol=1e-12, atol=1e-12)
        check = (t + 1) % period == 0
        cl, tail, due = dl.step_end(cl, tail, W, check)
        if due:
            keep = np.zeros((L, len(due), wl.hkv, wl.keep), dtype=np.int64)
            for l in range(L):
                q_win = dl.window_queries(rings[l], cl, due, W)
                for r, b in enumerate(due):
                    assert np.array_equal(q_win[r], np.array(dq[l][b][-W:]))
                    n = int(cl[b])
                    k_win = np.stack([np.stack([dk[l][b][g][s] for g in range(wl.hkv)])
                                      for s in range(n - W, n)])
                    sc = ok.window_scores(q_win[r].astype(np.float64), k_win.astype(np.float64),
                                          scale)
                    for g in range(wl.hkv):
                        sel = ok.select_topk(sc[g], wl.keep)
                        keep[l, r, g] = ok.token2chunk(sc[g], sel, ok.anchors_for(0.5, wl.keep),
                                                       8, 1)
            st, kp, vp, bt, cl2, fl, top, _ = ok.compact(kp, vp, bt, cl, fl, top, due, W, keep,
                                                        page)
            assert st == ok.OK
            for l in range(L):
                for r, b in enumerate(due):
                    n = int(cl[b])
                    for g in range(wl.hkv):
                        for rows in (dk[l][b], dv[l][b]):
                            rows[g] = rows[g][:n - W] + [rows[g][n - W + int(x)]
                                                         for x in keep[l, r, g]]
            assert all(int(cl2[b]) == int(cl[b]) - W + wl.keep for b in due)
            cl = cl2
            tail = dl.reset_tails(tail, due)
            compressions += len(due)
        # the paged cache equals the dense model, and every block is used once or free once
        for l in range(L):
            for b in range(wl.batch):
                assert len(dk[l][b][0]) == cl[b]
                for g in range(wl.hkv):
                    for s in range(int(cl[b])):
                        assert np.array_equal(paged_row(kp[l], bt, b, s, g, page), dk[l][b][g][s])
                        assert np.array_equal(paged_row(vp[l], bt, b, s, g, page), dv[l][b][g][s])
        used = [int(x) for x in bt[bt >= 0].ravel()]
        free = [int(x) for x in fl[:top]]
        assert sorted(used + free) == list(range(cache["num_blocks"]))
    return compressions


@pytest.mark.parametrize("period", [1, 7])
def test_loop_matches_dense_model(period):
    # 45 steps from contexts of 20..37 with W = 16: every sequence is compressed at least twice
    assert run_loop(LOOP, 3, 45, period) >= 2 * LOOP.batch


def test_step_begin_allocation_order_and_errors():
    bt = np.full((3, 4), -1, dtype=np.int64)
    bt[0, 0] = 10
    bt[1, 0] = 11
    bt[2, :2] = [12, 13]
    cl = np.array([16, 5, 32])
    fl = np.array([1, 2, 3, 4, 5, 0, 0])
    st, bt2, top = dl.step_begin(bt, cl, fl, 5, 16)
    assert st == dl.OK and top == 3
    assert bt2[0, 1] == 5 and bt2[2, 2] == 4           # ascending sequences, top of the stack
    assert np.array_equal(np.delete(bt2.ravel(), [1, 10]), np.delete(bt.ravel(), [1, 10]))
    st, bt3, top3 = dl.step_begin(bt, cl, fl, 1, 16)   # two needed, one free
    assert st == dl.ERR_OUT_OF_BLOCKS and top3 == 1 and np.array_equal(bt3, bt)
    st, bt4, _ = dl.step_begin(bt, np.array([64, 5, 32]), fl, 5, 16)   # past the table
    assert st == dl.ERR_INVALID_ARG and np.array_equal(bt4, bt)


def test_trigger_and_ring_rows():
    cl, tail, due = dl.step_end(np.array([10, 20, 30]), np.array([15, 3, 16]), 16, check=False)
    assert list(cl) == [11, 21, 31] and list(tail) == [16, 4, 17] and due == []
    _, _, due = dl.step_end(np.array([10, 20, 30]), np.array([15, 3, 16]), 16, check=True)
    assert due == [0, 2]
    # ring rows: slot s at s mod W and s mod W + W; the window [n-W, n) is contiguous
    W = 4
    ring = np.zeros((1, 2 * W, 1, 1))
    for s in range(6, 13):
        ring[0, s % W, 0, 0] = ring[0, s % W + W, 0, 0] = s
    win = dl.window_queries(ring, np.array([13]), [0], W)
    assert list(win[0, :, 0, 0]) == [9, 10, 11, 12]


def test_trigger_capacity():
    cl, tl, due = dl.step_end(np.array([38, 39, 40]), None, 0, check=True, capacity=40)
    assert tl is None and list(cl) == [39, 40, 41] and due == [1, 2]
    _, _, due = dl.step_end(np.array([38, 39, 40]), None, 0, check=False, capacity=40)
    assert due == []


LAC_LOOP = synth.Workload("lacloop", batch=3, layers=4, hq=4, hkv=2, head_dim=16, ctx_lo=20,
                          ctx_hi=35, window=0, keep=0, spare_blocks=4)
LAC = dict(span=2, overlap=1, rung=4, budget=24, sink=4, recent=4)


def test_lacache_loop_matches_dense_model():
    """LaCache inside the decode loop: at check steps every sequence that reached the capacity
    is laddered over its whole cache. The dense model keeps, per layer, the slots that
    ladder_keep_slots names, by list surgery."""
    wl, seed, steps, period = LAC_LOOP, 4, 60, 4
    assert ol.check_params(wl.layers, LAC["span"], LAC["overlap"], LAC["rung"], LAC["budget"],
                           LAC["sink"], LAC["recent"])
    cap = LAC["sink"] + LAC["recent"] + ol.region_capacity(wl.layers, LAC["span"], LAC["budget"],
                                                          LAC["sink"], LAC["recent"])
    cache = synth.make_cache(wl, seed, "cpu", with_queries=False, extra_pages=6)
    page, L, G = wl.page, wl.layers, wl.group
    scale = 1 / math.sqrt(wl.head_dim)
    kp = [np32(t) for t in cache["k"]]
    vp = [np32(t) for t in cache["v"]]
    bt = cache["block_table"].numpy().astype(np.int64)
    cl = cache["ctx_len"].numpy().astype(np.int64)
    fl = cache["free_list"].numpy().astype(np.int64)
    top = int(cache["free_top"][0])
    dk = [[[kp[l][bt[b, s // page], s % page] for s in range(cl[b])] for b in range(wl.batch)]
          for l in range(L)]
    dv = [[[vp[l][bt[b, s // page], s % page] for s in range(cl[b])] for b in range(wl.batch)]
          for l in range(L)]
    passes = 0
    for t in range(steps):
        st, bt, top = dl.step_begin(bt, cl, fl, top, page)
        assert st == dl.OK
        for l in range(L):
            inp = synth.decode_step_inputs(wl, seed, t, layers=L)[l]
            q, kn, vn = np32(inp["q"]), np32(inp["k"]), np32(inp["v"])
            out, kp[l], vp[l], _ = dl.decode_append(q, kn, vn, kp[l], vp[l], bt, cl, scale,
                                                    page, None, 1)
            for b in range(wl.batch):
                dk[l][b].append(kn[b])
                dv[l][b].append(vn[b])
                for h in range(wl.hq):
                    rows_k = [r[h // G] for r in dk[l][b]]
                    rows_v = [r[h // G] for r in dv[l][b]]
                    assert np.allclose(out[b, h], dense_attention(q[b, h], rows_k, rows_v, scale),
                                       rtol=1e-12, atol=1e-12)
        cl, _, due = dl.step_end(cl, None, 0, (t + 1) % period == 0, capacity=cap)
        assert all(int(cl[b]) >= cap for b in due)
        if due:
            st, kp, vp, bt, cl2, fl, top = ol.lacache_compact(
                kp, vp, bt, cl, fl, top, due, LAC["span"], LAC["overlap"], LAC["rung"],
                LAC["budget"], LAC["sink"], LAC["recent"], page)
            assert st == ol.OK
            for b in due:
                n = int(cl[b])
                for l in range(L):
                    slots = ol.ladder_keep_slots(n, L, LAC["span"], LAC["overlap"], LAC["rung"],
                                                 LAC["budget"], LAC["sink"], LAC["recent"])[l]
                    dk[l][b] = [dk[l][b][int(x)] for x in slots]
                    dv[l][b] = [dv[l][b][int(x)] for x in slots]
                assert int(cl2[b]) == LAC["budget"]
            cl = cl2
            passes += len(due)
        for l in range(L):
            for b in range(wl.batch):
                assert len(dk[l][b]) == cl[b]
                for s in range(int(cl[b])):
                    assert np.array_equal(kp[l][bt[b, s // page], s % page], dk[l][b][s])
                    assert np.array_equal(vp[l][bt[b, s // page], s % page], dv[l][b][s])
        used = [int(x) for x in bt[bt >= 0].ravel()]
        assert sorted(used + [int(x) for x in fl[:top]]) == list(range(cache["num_blocks"]))
    assert passes >= 2 * wl.batch       # every sequence laddered at least twice
