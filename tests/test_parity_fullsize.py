"""Parity at full size, in the launch configuration bench.py times.

The one-layer workload (batch 32, 28 q / 4 kv heads, d=128, 4096-token caches, W=1024, k=204)
goes through bench.Step: kara_score -> kara_select_chunks (selection and Token2Chunk in one
kernel, both written) -> kara_compact -> paged_decode_attn. Checked against the oracle: every
score row elementwise (the scorer's cluster ranges end inside items here, so the split-item
sum is element-checked too), selection and Token2Chunk exactly on every row, compaction
bit-exact on every sequence, decode on every (sequence, query head).

The step workload (28 layers, batch 128, ragged 2K-16K contexts, W=1024, k=204), the bench's
headline configuration, goes through the same Step; it is too large for the oracle to redo
whole, so: the W*G row sums of every score row, sampled score rows elementwise, selection and
Token2Chunk exactly on sampled rows, the block table / lengths / free list exactly (the
oracle's bookkeeping of all 28 layers), every moved K/V row of sampled (layer, sequence) pairs
bit-exact, and decode on sampled (layer, sequence) pairs.

The LaCache ladder runs at its workload's sequence length (64K tokens, 32 layers, 8 KV heads)
with a reduced batch and is checked on sampled layers.
"""

import math

import numpy as np
import pytest
import torch

import bench
from decode_kv_cache_kara_b200 import kara as K
from decode_kv_cache_kara_b200 import synth
from oracle import decode as od
from oracle import kara as ok
from oracle import lacache as ol
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def layer_step():
    wl = bench.LAYER_WORKLOAD
    cache = synth.make_cache(wl, 1234 + 1, "cuda")
    before = {
        "k": H.bits(cache["k"][0]), "v": H.bits(cache["v"][0]),
        "q_win": cache["q_win"][0].cpu(), "q_dec": cache["q_dec"].cpu(),
        "block_table": H.i32(cache["block_table"]), "ctx_len": H.i32(cache["ctx_len"]),
        "free_list": H.i32(cache["free_list"]), "free_top": int(cache["free_top"][0]),
    }
    step = bench.Step(cache, wl)
    n0 = K.kara_launch_count()
    K.kara_score(cache["q_win"][0], cache["k"][0], step.pool, wl.window,
                 scores=step.scores[0], workspace=step.ws, status=step.status)
    score_launches = K.kara_launch_count() - n0
    step.run(restore=False)
    torch.cuda.synchronize()
    assert K.read_status(step.status) == 0
    yield wl, cache, step, before, score_launches
    del step, cache
    torch.cuda.empty_cache()


def _pool_f64(bits):
    return torch.from_numpy(bits).view(torch.bfloat16).double().numpy()


def test_fullsize_scores_every_row(layer_step):
    wl, cache, step, before, score_launches = layer_step
    # 7168 (item, tile) pairs over the resident clusters of 8 CTAs: ranges end inside items,
    # so the fused kernel is followed by the split-item sum (two launches)
    assert score_launches == 2
    scores = H.f64(step.scores[0])
    assert np.allclose(scores.sum(-1), wl.window * wl.group, rtol=1e-4)
    kf = _pool_f64(before["k"])
    scale = 1 / math.sqrt(wl.head_dim)
    for r in range(wl.batch):
        n = int(before["ctx_len"][r])
        slots = ok.window_slots(n, wl.window)
        kw = ok.gather_rows(kf, before["block_table"][r], slots, wl.page)
        qw = before["q_win"][r].double().numpy()
        H.assert_scores_close(scores[r], ok.window_scores(qw, kw, scale))


def test_fullsize_select_and_token2chunk_every_row(layer_step):
    wl, cache, step, before, _ = layer_step
    scores = H.f64(step.scores[0])
    sel = H.i32(step.sel[0])
    keep = H.i32(step.keep[0])
    na = ok.anchors_for(wl.anchor_frac, wl.keep)
    for r in range(wl.batch):
        for g in range(wl.hkv):
            assert np.array_equal(sel[r, g], ok.select_topk(scores[r, g], wl.keep))
            assert np.array_equal(keep[r, g], ok.token2chunk(scores[r, g], sel[r, g], na,
                                                             wl.gap_limit, wl.widen))


def test_fullsize_compaction_bit_exact(layer_step):
    wl, cache, step, before, _ = layer_step
    keep = H.i32(step.keep)
    st, kp, vp, bt, cl, fl, top, _ = ok.compact(
        [before["k"]], [before["v"]], before["block_table"], before["ctx_len"],
        before["free_list"], before["free_top"], list(range(wl.batch)), wl.window, keep, wl.page)
    assert st == ok.OK
    assert np.array_equal(H.i32(cache["block_table"]), bt)
    assert np.array_equal(H.i32(cache["ctx_len"]), cl)
    assert int(cache["free_top"][0]) == top
    assert np.array_equal(H.i32(cache["free_list"])[:top], fl[:top])
    kg, vg = H.bits(cache["k"][0]), H.bits(cache["v"][0])
    for b in range(wl.batch):
        n = int(cl[b])
        assert np.array_equal(H.logical_rows(kg, bt[b], n), H.logical_rows(kp[0], bt[b], n))
        assert np.array_equal(H.logical_rows(vg, bt[b], n), H.logical_rows(vp[0], bt[b], n))


def test_fullsize_decode_every_sequence(layer_step):
    wl, cache, step, before, _ = layer_step
    out = H.f64(step.out[0])
    bt, cl = H.i32(cache["block_table"]), H.i32(cache["ctx_len"])
    kf, vf = H.f64(cache["k"][0]), H.f64(cache["v"][0])
    q = before["q_dec"].double().numpy()
    ref = od.decode_attention(q, kf, vf, bt, cl, 1 / math.sqrt(wl.head_dim), wl.page)
    assert np.allclose(out, ref, atol=2e-2, rtol=1e-2)


# ------------------------------------------------------------------------------------------
# the step workload (the bench's headline configuration), sampled
# ------------------------------------------------------------------------------------------
@pytest.fixture(scope="module")
def full_step():
    wl = bench.WORKLOAD
    cache = synth.make_cache(wl, bench.rank_seed(0), "cuda")
    bt0, cl0 = H.i32(cache["block_table"]), H.i32(cache["ctx_len"])
    fl0, top0 = H.i32(cache["free_list"]), int(cache["free_top"][0])
    step = bench.Step(cache, wl)
    step.run(restore=False)
    torch.cuda.synchronize()
    assert K.read_status(step.status) == 0
    yield wl, cache, step, (bt0, cl0, fl0, top0)
    del step, cache
    torch.cuda.empty_cache()


def _window_rows(pool, table_row, slots, page=16):
    """K or V rows [len(slots), Hkv, d] of one sequence from a device pool, as float64."""
    idx = torch.as_tensor(table_row[slots // page], device=pool.device)
    rows = torch.as_tensor(slots % page, device=pool.device)
    return pool[idx, rows].double().cpu().numpy()


def test_step_workload_scores_sampled(full_step):
    wl, cache, step, (bt0, cl0, _, _) = full_step
    sums = step.scores.double().sum(-1).cpu().numpy()          # [L, B, Hkv]
    assert np.allclose(sums, wl.window * wl.group, rtol=1e-4)
    rng = np.random.default_rng(5)
    scale = 1 / math.sqrt(wl.head_dim)
    # random rows, plus the last row (its items go to the helper beside the fused kernel when
    # the clusters leave SMs idle) and the first
    picks = list(zip(rng.integers(0, wl.layers, 4), rng.integers(0, wl.batch, 4)))
    picks += [(wl.layers - 1, wl.batch - 1), (0, 0)]
    for layer, r in picks:
        slots = ok.window_slots(int(cl0[r]), wl.window)
        kw = _window_rows(cache["k"][layer], bt0[r], slots)    # old rows, still in place
        qw = cache["q_win"][layer][r].double().cpu().numpy()
        H.assert_scores_close(H.f64(step.scores[layer, r]), ok.window_scores(qw, kw, scale))


def test_step_workload_select_and_token2chunk_sampled(full_step):
    wl, cache, step, _ = full_step
    na = ok.anchors_for(wl.anchor_frac, wl.keep)
    rng = np.random.default_rng(6)
    for layer, r, g in zip(rng.integers(0, wl.layers, 48), rng.integers(0, wl.batch, 48),
                           rng.integers(0, wl.hkv, 48)):
        s = H.f64(step.scores[layer, r, g])
        sel = ok.select_topk(s, wl.keep)
        assert np.array_equal(H.i32(step.sel[layer, r, g]), sel)
        assert np.array_equal(H.i32(step.keep[layer, r, g]),
                              ok.token2chunk(s, sel, na, wl.gap_limit, wl.widen))


def test_step_workload_compaction(full_step):
    wl, cache, step, (bt0, cl0, fl0, top0) = full_step
    keep = H.i32(step.keep)
    # the bookkeeping of all layers, exactly (the oracle with no pools moves no rows)
    st, _, _, bt, cl, fl, top, fresh = ok.compact([], [], bt0, cl0, fl0, top0,
                                                  list(range(wl.batch)), wl.window, keep,
                                                  wl.page)
    assert st == ok.OK
    assert np.array_equal(H.i32(cache["block_table"]), bt)
    assert np.array_equal(H.i32(cache["ctx_len"]), cl)
    assert int(cache["free_top"][0]) == top
    assert np.array_equal(H.i32(cache["free_list"])[:top], fl[:top])
    # the rows of sampled (layer, sequence) pairs, bit-exact: the prefix of the first window
    # page and the kept rows of every KV head, read through the new table, against the old
    # rows (which compaction left in place)
    rng = np.random.default_rng(7)
    for layer, b in zip(rng.integers(0, wl.layers, 6), rng.integers(0, wl.batch, 6)):
        start = int(cl0[b]) - wl.window
        p0 = start // wl.page
        for pool in (cache["k"][layer], cache["v"][layer]):
            pre_new = torch.as_tensor(np.arange(p0 * wl.page, start))
            new_rows = _window_rows(pool, bt[b], np.arange(p0 * wl.page, start + wl.keep))
            old_pre = _window_rows(pool, bt0[b], pre_new.numpy())
            assert np.array_equal(new_rows[:len(pre_new)], old_pre)
            for g in range(wl.hkv):
                old = _window_rows(pool, bt0[b], start + keep[layer, b, g])[:, g]
                assert np.array_equal(new_rows[len(pre_new):, g], old)


def test_step_workload_decode_sampled(full_step):
    wl, cache, step, _ = full_step
    bt, cl = H.i32(cache["block_table"]), H.i32(cache["ctx_len"])
    rng = np.random.default_rng(8)
    scale = 1 / math.sqrt(wl.head_dim)
    for layer, b in zip(rng.integers(0, wl.layers, 4), rng.integers(0, wl.batch, 4)):
        n = int(cl[b])
        kk = _window_rows(cache["k"][layer], bt[b], np.arange(n))
        vv = _window_rows(cache["v"][layer], bt[b], np.arange(n))
        q = step.q_dec[layer][b:b + 1].double().cpu().numpy()
        ref = od.decode_attention(q, kk[None], vv[None], np.array([[0]]), np.array([n]), scale, n)
        assert np.allclose(H.f64(step.out[layer, b]), ref[0], atol=2e-2, rtol=1e-2)


# ------------------------------------------------------------------------------------------
# LaCache at its workload's sequence length
# ------------------------------------------------------------------------------------------
def test_lacache_full_length_sampled_layers():
    ex = synth.WORKLOADS["lacache"].extra
    wl = synth.WORKLOADS["lacache"].with_(batch=1)
    cache = synth.make_cache(wl, 1234 + 4, "cuda", with_queries=False)
    sample = [0, 13, 31]
    before = {layer: (H.bits(cache["k"][layer]), H.bits(cache["v"][layer])) for layer in sample}
    bt0, cl0 = H.i32(cache["block_table"]), H.i32(cache["ctx_len"])
    pool = K.PagedPool.from_cache(cache)
    status = K.lacache_compact(cache["k"], cache["v"], pool, ex["span"], ex["overlap"], ex["rung"],
                               ex["budget"], ex["sink"], ex["recent"])
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    bt, cl = H.i32(cache["block_table"]), H.i32(cache["ctx_len"])
    assert int(cl[0]) == ex["budget"]
    n = int(cl0[0])
    keep = ol.ladder_keep_slots(n, wl.layers, ex["span"], ex["overlap"], ex["rung"], ex["budget"],
                                ex["sink"], ex["recent"])
    for layer in sample:
        kb, vb = before[layer]
        new_k = H.logical_rows(H.bits(cache["k"][layer]), bt[0], ex["budget"])
        new_v = H.logical_rows(H.bits(cache["v"][layer]), bt[0], ex["budget"])
        src = keep[layer]
        assert np.array_equal(new_k, kb[bt0[0][src // 16], src % 16])
        assert np.array_equal(new_v, vb[bt0[0][src // 16], src % 16])
