"""GPU parity of the decode loop (kara_step_begin, kara_decode_append, kara_step_end, and at
check steps kara_score_ring, kara_select, kara_token2chunk, kara_compact, kara_reset_tails)
against the decode-loop oracle, step by step on the same seeded inputs.

Checks: every step's attention outputs (2e-2 abs / 1e-2 rel, bf16 output of fp32 arithmetic);
the due lists exactly; the ring scores within the score tolerance (1e-3 rel); select and
Token2Chunk exactly on the GPU's scores (identical inputs); after every compression and at
the end, the block table, lengths, free list and top, every cached K/V row and the query rings
bit-exact. The oracle compresses with the GPU's keep sets (equal to its own on those scores),
so both sides stay in lockstep.
"""

import math

import numpy as np
import pytest
import torch

from decode_kv_cache_kara_b200 import kara as K
from decode_kv_cache_kara_b200 import synth
from oracle import decode_loop as dl
from oracle import kara as ok
from tests import helpers as H

pytestmark = pytest.mark.gpu

CASES = {
    # W = 128: the fused cluster scorer (one CTA per cluster); G = 4, d = 64
    "w128_fused": (synth.Workload("loop128", batch=3, layers=2, hq=8, hkv=2, head_dim=64,
                                  ctx_lo=20, ctx_hi=40, window=128, keep=26, spare_blocks=4),
                   16, 300),
    # W = 64: the fused scorer with one CTA owning 64 keys and half-empty query tiles, reading
    # the window-query ring; G = 2, d = 128, a check every 8 steps
    "w64_partial": (synth.Workload("loop64", batch=3, layers=2, hq=4, hkv=2, head_dim=128,
                                   ctx_lo=17, ctx_hi=50, window=64, keep=13, spare_blocks=4),
                    8, 150),
}


def f32(t):
    return t.float().cpu().numpy()


def rows_equal(gpu_pool, ref_pool, bt, cl, page):
    for b in range(len(cl)):
        for s in range(int(cl[b])):
            blk = int(bt[b, s // page])
            if not np.array_equal(gpu_pool[blk, s % page], ref_pool[blk, s % page]):
                return False
    return True


@pytest.mark.parametrize("name", list(CASES))
def test_decode_loop_matches_oracle(name):
    wl, period, steps = CASES[name]
    seed = 21
    W, L, page = wl.window, wl.layers, wl.page
    scale = 1 / math.sqrt(wl.head_dim)
    na = wl.anchor_frac
    cpu = synth.make_cache(wl, seed, "cpu", with_queries=False, extra_pages=steps // page + 2)
    dev = H.to_device(cpu)
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    tail = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    due = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    due_count = torch.zeros(1, dtype=torch.int32, device="cuda")
    rings = [torch.zeros((wl.batch, 2 * W, wl.hq, wl.head_dim), dtype=torch.bfloat16,
                         device="cuda") for _ in range(L)]
    # oracle state
    kp = [f32(t) for t in cpu["k"]]
    vp = [f32(t) for t in cpu["v"]]
    bt, cl = H.i32(cpu["block_table"]), H.i32(cpu["ctx_len"])
    fl, top = H.i32(cpu["free_list"]), int(cpu["free_top"][0])
    otail = np.zeros(wl.batch, dtype=np.int64)
    orings = [np.zeros((wl.batch, 2 * W, wl.hq, wl.head_dim), dtype=np.float32) for _ in range(L)]

    def check_state():
        assert np.array_equal(H.i32(dev["block_table"]), bt)
        assert np.array_equal(H.i32(dev["ctx_len"]), cl)
        assert int(dev["free_top"][0]) == top
        assert np.array_equal(H.i32(dev["free_list"])[:top], fl[:top])
        for layer in range(L):
            assert rows_equal(f32(dev["k"][layer]), kp[layer], bt, cl, page)
            assert rows_equal(f32(dev["v"][layer]), vp[layer], bt, cl, page)

    compressions = 0
    for t in range(steps):
        K.kara_step_begin(pool, status)
        st, bt, top = dl.step_begin(bt, cl, fl, top, page)
        assert st == dl.OK
        inputs = synth.decode_step_inputs(wl, seed, t)
        for layer in range(L):
            q, kn, vn = (inputs[layer][x].cuda() for x in ("q", "k", "v"))
            out = K.kara_decode_append(q, kn, vn, dev["k"][layer], dev["v"][layer], pool,
                                       rings[layer], W, status=status)
            ref, kp[layer], vp[layer], orings[layer] = dl.decode_append(
                f32(q), f32(kn), f32(vn), kp[layer], vp[layer], bt, cl, scale, page,
                orings[layer], W)
            assert np.allclose(H.f64(out), ref, atol=2e-2, rtol=1e-2), (t, layer)
        check = (t + 1) % period == 0
        K.kara_step_end(pool, tail, W, check, due, due_count)
        cl, otail, odue = dl.step_end(cl, otail, W, check)
        if not check:
            continue
        torch.cuda.synchronize()
        assert K.read_status(status) == 0
        cnt = int(due_count[0])
        assert list(H.i32(due)[:cnt]) == odue
        if cnt == 0:
            continue
        seq = due[:cnt]
        keep = torch.empty((L, cnt, wl.hkv, wl.keep), dtype=torch.int32, device="cuda")
        scores = []
        for layer in range(L):
            sc = K.kara_score_ring(rings[layer], dev["k"][layer], pool, W, seq, cnt,
                                   status=status)
            sel = K.kara_select(sc, wl.keep)
            K.kara_token2chunk(sc, sel, na, wl.gap_limit, wl.widen, keep=keep[layer])
            scores.append(sc)
        K.kara_compact(dev["k"], dev["v"], pool, W, keep, seq_ids=seq, status=status)
        K.kara_reset_tails(tail, seq, cnt)
        torch.cuda.synchronize()
        assert K.read_status(status) == 0
        kk = H.i32(keep)
        for layer in range(L):
            qwin = dl.window_queries(orings[layer], cl, odue, W).astype(np.float64)
            s_gpu = H.f64(scores[layer])
            for r, b in enumerate(odue):
                n = int(cl[b])
                kw = np.stack([kp[layer][bt[b, s // page], s % page] for s in range(n - W, n)])
                H.assert_scores_close(s_gpu[r], ok.window_scores(qwin[r], kw.astype(np.float64),
                                                                 scale))
                for g in range(wl.hkv):
                    sel = ok.select_topk(s_gpu[r, g], wl.keep)
                    assert np.array_equal(kk[layer, r, g],
                                          ok.token2chunk(s_gpu[r, g], sel,
                                                         ok.anchors_for(na, wl.keep),
                                                         wl.gap_limit, wl.widen))
        st, kp, vp, bt, cl, fl, top, _ = ok.compact(kp, vp, bt, cl, fl, top, odue, W, kk, page)
        assert st == ok.OK
        otail = dl.reset_tails(otail, odue)
        assert np.array_equal(H.i32(tail), otail)
        check_state()
        compressions += cnt
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    check_state()
    for layer in range(L):
        assert np.array_equal(f32(rings[layer]), orings[layer])
    assert compressions >= 2 * wl.batch


def test_step_begin_out_of_blocks_changes_nothing():
    wl = synth.Workload("oob", batch=4, layers=1, hq=2, hkv=1, head_dim=64, ctx_lo=32,
                        ctx_hi=32, window=16, keep=4)
    dev = H.to_device(synth.make_cache(wl, 5, "cpu", with_queries=False, extra_pages=1))
    dev["free_top"].fill_(2)            # four sequences at a page boundary, two free blocks
    before = H.i32(dev["block_table"]).copy()
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    K.kara_step_begin(pool, status)
    torch.cuda.synchronize()
    assert K.read_status(status) == K.ERR_OUT_OF_BLOCKS
    assert np.array_equal(H.i32(dev["block_table"]), before)
    assert int(dev["free_top"][0]) == 2


def test_lacache_loop_matches_oracle():
    """LaCache inside the decode loop: at check steps the sequences whose length reached the
    capacity sink + recent + R_max are laddered over their whole cache (lacache_compact), then
    decoding goes on; every sequence is laddered at least twice. Outputs, due lists and the
    whole cache state in lockstep with the oracle."""
    from oracle import lacache as ol
    wl = synth.Workload("lacloop", batch=3, layers=4, hq=4, hkv=2, head_dim=64, ctx_lo=20,
                        ctx_hi=35, window=0, keep=0, spare_blocks=4)
    lac = dict(span=2, overlap=1, rung=4, budget=24, sink=4, recent=4)
    seed, steps, period, page, L = 4, 60, 4, wl.page, wl.layers
    cap = lac["sink"] + lac["recent"] + ol.region_capacity(L, lac["span"], lac["budget"],
                                                          lac["sink"], lac["recent"])
    scale = 1 / math.sqrt(wl.head_dim)
    cpu = synth.make_cache(wl, seed, "cpu", with_queries=False, extra_pages=6)
    dev = H.to_device(cpu)
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    due = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    due_count = torch.zeros(1, dtype=torch.int32, device="cuda")
    kp = [f32(t) for t in cpu["k"]]
    vp = [f32(t) for t in cpu["v"]]
    bt, cl = H.i32(cpu["block_table"]), H.i32(cpu["ctx_len"])
    fl, top = H.i32(cpu["free_list"]), int(cpu["free_top"][0])
    passes = 0
    for t in range(steps):
        K.kara_step_begin(pool, status)
        st, bt, top = dl.step_begin(bt, cl, fl, top, page)
        assert st == dl.OK
        inputs = synth.decode_step_inputs(wl, seed, t)
        for layer in range(L):
            q, kn, vn = (inputs[layer][x].cuda() for x in ("q", "k", "v"))
            out = K.kara_decode_append(q, kn, vn, dev["k"][layer], dev["v"][layer], pool,
                                       status=status)
            ref, kp[layer], vp[layer], _ = dl.decode_append(f32(q), f32(kn), f32(vn), kp[layer],
                                                            vp[layer], bt, cl, scale, page, None, 1)
            assert np.allclose(H.f64(out), ref, atol=2e-2, rtol=1e-2), (t, layer)
        check = (t + 1) % period == 0
        K.kara_step_end(pool, None, 0, check, due, due_count, capacity=cap)
        cl, _, odue = dl.step_end(cl, None, 0, check, capacity=cap)
        if not check:
            continue
        torch.cuda.synchronize()
        cnt = int(due_count[0])
        assert list(H.i32(due)[:cnt]) == odue
        if cnt == 0:
            continue
        K.lacache_compact(dev["k"], dev["v"], pool, lac["span"], lac["overlap"], lac["rung"],
                          lac["budget"], lac["sink"], lac["recent"], seq_ids=due[:cnt],
                          status=status)
        torch.cuda.synchronize()
        assert K.read_status(status) == 0
        st, kp, vp, bt, cl, fl, top = ol.lacache_compact(
            kp, vp, bt, cl, fl, top, odue, lac["span"], lac["overlap"], lac["rung"],
            lac["budget"], lac["sink"], lac["recent"], page)
        assert st == ol.OK
        assert np.array_equal(H.i32(dev["block_table"]), bt)
        assert np.array_equal(H.i32(dev["ctx_len"]), cl)
        assert int(dev["free_top"][0]) == top
        assert np.array_equal(H.i32(dev["free_list"])[:top], fl[:top])
        for layer in range(L):
            assert rows_equal(f32(dev["k"][layer]), kp[layer], bt, cl, page)
            assert rows_equal(f32(dev["v"][layer]), vp[layer], bt, cl, page)
        passes += cnt
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    assert passes >= 2 * wl.batch


def test_decode_append_empty_context_and_no_ring():
    """A sequence with an empty cache: its block comes from kara_step_begin, the new token is
    the only one, so the output is its V row (bf16, exactly); no ring is passed, and a step
    end without a check only advances the lengths."""
    wl = synth.Workload("empty", batch=3, layers=1, hq=4, hkv=2, head_dim=128, ctx_lo=20,
                        ctx_hi=40, window=16, keep=4)
    cpu = synth.make_cache(wl, 13, "cpu", with_queries=False, extra_pages=2)
    cpu["ctx_len"][1] = 0
    cpu["block_table"][1].fill_(-1)
    # the emptied sequence's old blocks stay out of the free list (they are simply unused)
    dev = H.to_device(cpu)
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    K.kara_step_begin(pool, status)
    inp = synth.decode_step_inputs(wl, 13, 0)[0]
    q, kn, vn = (inp[x].cuda() for x in ("q", "k", "v"))
    out = K.kara_decode_append(q, kn, vn, dev["k"][0], dev["v"][0], pool, status=status)
    K.kara_step_end(pool)
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    assert int(dev["ctx_len"][1]) == 1 and int(dev["ctx_len"][0]) == int(cpu["ctx_len"][0]) + 1
    g_of_h = torch.arange(wl.hq) // wl.group
    assert torch.equal(out[1].cpu(), vn[1].cpu()[g_of_h])
    blk = int(dev["block_table"][1, 0])
    assert blk >= 0
    assert torch.equal(dev["k"][0][blk, 0].cpu(), kn[1].cpu())
    assert torch.equal(dev["v"][0][blk, 0].cpu(), vn[1].cpu())
    # the other sequences against the oracle
    scale = 1 / math.sqrt(wl.head_dim)
    bt = H.i32(dev["block_table"])
    ref, _, _, _ = dl.decode_append(f32(q), f32(kn), f32(vn), f32(cpu["k"][0]), f32(cpu["v"][0]),
                                    bt, H.i32(cpu["ctx_len"]), scale, wl.page, None, 1)
    assert np.allclose(H.f64(out), ref, atol=2e-2, rtol=1e-2)
