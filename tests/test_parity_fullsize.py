"""Parity at full size, in the launch configuration bench.py times.

The layer workload (batch 32, 28 q / 4 kv heads, d=128, 4096-token caches, W=1024, k=204) goes
through the same calls as one bench step (bench.Step): kara_score -> kara_select_chunks
(selection and Token2Chunk in one kernel, both written) -> kara_compact -> paged_decode_attn. Checks: sampled score rows against the
oracle, and the W*G row sums on every row; select and Token2Chunk exactly on sampled rows;
compaction bit-exact on every sequence; decode on sampled (sequence, query head) pairs. The
LaCache ladder runs at its workload's sequence length (64K tokens, 32 layers, 8 KV heads) with
a reduced batch and is checked on sampled layers.
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
    wl = bench.WORKLOAD
    cache = synth.make_cache(wl, bench.rank_seed(0), "cuda")
    before = {
        "k": H.bits(cache["k"][0]), "v": H.bits(cache["v"][0]),
        "q_win": cache["q_win"][0].cpu(), "q_dec": cache["q_dec"].cpu(),
        "block_table": H.i32(cache["block_table"]), "ctx_len": H.i32(cache["ctx_len"]),
        "free_list": H.i32(cache["free_list"]), "free_top": int(cache["free_top"][0]),
    }
    step = bench.Step(cache, wl)
    step.run(restore=False)
    torch.cuda.synchronize()
    assert K.read_status(step.status) == 0
    return wl, cache, step, before


def _pool_f64(bits):
    return torch.from_numpy(bits).view(torch.bfloat16).double().numpy()


def test_fullsize_scores_sampled_rows(layer_step):
    wl, cache, step, before = layer_step
    scores = H.f64(step.scores)
    assert np.allclose(scores.sum(-1), wl.window * wl.group, rtol=1e-4)
    kf = _pool_f64(before["k"])
    rng = np.random.default_rng(0)
    for r, g in zip(rng.integers(0, wl.batch, 3), rng.integers(0, wl.hkv, 3)):
        n = int(before["ctx_len"][r])
        slots = ok.window_slots(n, wl.window)
        kw = ok.gather_rows(kf, before["block_table"][r], slots, wl.page)[:, g:g + 1]
        heads = list(range(g * wl.group, (g + 1) * wl.group))
        qw = before["q_win"][r][:, heads].double().numpy()
        ref = ok.window_scores(qw, kw, 1 / math.sqrt(wl.head_dim))[0]
        H.assert_scores_close(scores[r, g], ref)


def test_fullsize_select_and_token2chunk_sampled_rows(layer_step):
    wl, cache, step, before = layer_step
    scores = H.f64(step.scores)
    sel = H.i32(step.sel)
    keep = H.i32(step.keep[0])
    na = ok.anchors_for(wl.anchor_frac, wl.keep)
    rng = np.random.default_rng(1)
    for r, g in zip(rng.integers(0, wl.batch, 8), rng.integers(0, wl.hkv, 8)):
        assert np.array_equal(sel[r, g], ok.select_topk(scores[r, g], wl.keep))
        assert np.array_equal(keep[r, g], ok.token2chunk(scores[r, g], sel[r, g], na,
                                                         wl.gap_limit, wl.widen))


def test_fullsize_compaction_bit_exact(layer_step):
    wl, cache, step, before = layer_step
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


def test_fullsize_decode_sampled_pairs(layer_step):
    wl, cache, step, before = layer_step
    out = H.f64(step.out)
    bt, cl = H.i32(cache["block_table"]), H.i32(cache["ctx_len"])
    kf, vf = H.f64(cache["k"][0]), H.f64(cache["v"][0])
    q = before["q_dec"].double().numpy()
    rng = np.random.default_rng(2)
    for b in rng.integers(0, wl.batch, 4):
        ref = od.decode_attention(q[b:b + 1], kf, vf, bt[b:b + 1], cl[b:b + 1],
                                  1 / math.sqrt(wl.head_dim), wl.page)
        assert np.allclose(out[b], ref[0], atol=2e-2, rtol=1e-2)


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
