"""GPU parity of the variants the pages leave open: the mean and max aggregations of the
window scores (kara_score_ex) and a selection shared across the KV heads of a layer
(kara_sum_heads, kara_select / kara_token2chunk on the head sums, kara_expand_keep).

Tolerances: scores 1e-3 relative (+1e-6 absolute), as the sum; the head sums equal an fp32
sum in ascending head order; selection, Token2Chunk and the expanded keep sets exact given the
same scores; compaction with the shared keep sets bit-exact.
"""

import math

import numpy as np
import pytest
import torch

from decode_kv_cache_kara_b200 import kara as K
from decode_kv_cache_kara_b200 import synth
from oracle import kara as ok
from tests import helpers as H

pytestmark = pytest.mark.gpu

LAYER = synth.WORKLOADS["layer"]
CASES = {
    "w512_fused": LAYER.with_(batch=3, ctx_lo=520, ctx_hi=900, window=512, keep=102),
    "w200_twopass": LAYER.with_(batch=3, ctx_lo=300, ctx_hi=700, window=200, keep=40),
}
AGGS = {"mean": K.AGG_MEAN, "max": K.AGG_MAX}


def oracle_agg(cpu, wl, agg):
    q = H.f64(cpu["q_win"][0])
    kf = H.f64(cpu["k"][0])
    bt, cl = H.i32(cpu["block_table"]), H.i32(cpu["ctx_len"])
    scale = 1 / math.sqrt(wl.head_dim)
    out = []
    for r in range(wl.batch):
        slots = ok.window_slots(int(cl[r]), wl.window)
        kw = ok.gather_rows(kf, bt[r], slots, wl.page)
        out.append(ok.window_scores_agg(q[r], kw, scale, agg))
    return np.stack(out)


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("agg", list(AGGS))
def test_score_aggregation_matches_oracle(name, agg):
    wl = CASES[name]
    cpu, dev = H.make(wl, 8)
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    sc = K.kara_score_ex(dev["q_win"][0], dev["k"][0], pool, wl.window, agg=AGGS[agg],
                         status=status)
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    H.assert_scores_close(H.f64(sc), oracle_agg(cpu, wl, agg))
    if agg == "mean":   # the mean of each (sequence, KV head) row sums to 1
        assert np.allclose(H.f64(sc).sum(-1), 1.0, rtol=1e-4)


def test_max_from_the_ring_equals_max_from_q_win():
    """The ring form reads the same query rows: the same tiles, the same result, bit for bit."""
    wl = CASES["w200_twopass"]
    cpu, dev = H.make(wl, 9)
    pool = K.PagedPool.from_cache(dev)
    W = wl.window
    ring = torch.randn((wl.batch, 2 * W, wl.hq, wl.head_dim), device="cuda").to(torch.bfloat16)
    for b in range(wl.batch):
        off = (int(cpu["ctx_len"][b]) - W) % W
        ring[b, off:off + W] = dev["q_win"][0][b]
    seq = torch.arange(wl.batch, dtype=torch.int32, device="cuda")
    a = K.kara_score_ex(dev["q_win"][0], dev["k"][0], pool, W, agg=K.AGG_MAX)
    b = K.kara_score_ex(ring, dev["k"][0], pool, W, agg=K.AGG_MAX, ring=True, seq_ids=seq)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_shared_selection_across_kv_heads():
    wl = LAYER.with_(batch=3, ctx_lo=600, ctx_hi=900, window=256, keep=52, layers=2)
    cpu, dev = H.make(wl, 10)
    pool = K.PagedPool.from_cache(dev)
    na = wl.anchor_frac
    status = K.new_status()
    keep = torch.empty((wl.layers, wl.batch, wl.hkv, wl.keep), dtype=torch.int32, device="cuda")
    sums, shared = [], []
    for layer in range(wl.layers):
        sc = K.kara_score(dev["q_win"][layer], dev["k"][layer], pool, wl.window, status=status)
        tot = K.kara_sum_heads(sc)
        sel = K.kara_select(tot, wl.keep)
        ks = K.kara_token2chunk(tot, sel, na, wl.gap_limit, wl.widen)
        K.kara_expand_keep(ks, wl.hkv, keep=keep[layer])
        sums.append((sc, tot))
        shared.append(ks)
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    for layer in range(wl.layers):
        sc = sums[layer][0].cpu().numpy()
        ref = sc[:, 0].copy()
        for g in range(1, wl.hkv):
            ref = (ref + sc[:, g]).astype(np.float32)
        assert np.array_equal(sums[layer][1].cpu().numpy(), ref)
        for r in range(wl.batch):
            # selection and Token2Chunk of the oracle on the same (fp32) head sums
            tot = sums[layer][1][r].double().cpu().numpy()
            own = ok.token2chunk(tot, ok.select_topk(tot, wl.keep), ok.anchors_for(na, wl.keep),
                                 wl.gap_limit, wl.widen)
            assert np.array_equal(H.i32(shared[layer][r]), own)
            assert all(np.array_equal(H.i32(keep[layer, r, g]), own) for g in range(wl.hkv))
    # compaction with the shared keep sets, bit-exact against the oracle
    kb = [H.bits(t) for t in cpu["k"]]
    vb = [H.bits(t) for t in cpu["v"]]
    bt0, cl0 = H.i32(cpu["block_table"]), H.i32(cpu["ctx_len"])
    fl0, top0 = H.i32(cpu["free_list"]), int(cpu["free_top"][0])
    K.kara_compact(dev["k"], dev["v"], pool, wl.window, keep, status=status)
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    st, kpo, vpo, bt, cl, fl, top, _ = ok.compact(kb, vb, bt0, cl0, fl0, top0,
                                                  list(range(wl.batch)), wl.window, H.i32(keep),
                                                  wl.page)
    assert st == ok.OK
    assert np.array_equal(H.i32(dev["block_table"]), bt)
    assert np.array_equal(H.i32(dev["ctx_len"]), cl)
    for layer in range(wl.layers):
        kg, vg = H.bits(dev["k"][layer]), H.bits(dev["v"][layer])
        for b in range(wl.batch):
            n = int(cl[b])
            assert np.array_equal(H.logical_rows(kg, bt[b], n), H.logical_rows(kpo[layer], bt[b], n))
            assert np.array_equal(H.logical_rows(vg, bt[b], n), H.logical_rows(vpo[layer], bt[b], n))


def test_mean_from_the_ring_equals_mean_from_q_win_and_one_head_sums():
    wl = CASES["w512_fused"]
    cpu, dev = H.make(wl, 14)
    pool = K.PagedPool.from_cache(dev)
    W = wl.window
    ring = torch.zeros((wl.batch, 2 * W, wl.hq, wl.head_dim), device="cuda", dtype=torch.bfloat16)
    for b in range(wl.batch):
        off = (int(cpu["ctx_len"][b]) - W) % W
        ring[b, off:off + W] = dev["q_win"][0][b]
    seq = torch.arange(wl.batch, dtype=torch.int32, device="cuda")
    a = K.kara_score_ex(dev["q_win"][0], dev["k"][0], pool, W, agg=K.AGG_MEAN)
    b = K.kara_score_ex(ring, dev["k"][0], pool, W, agg=K.AGG_MEAN, ring=True, seq_ids=seq)
    one = K.kara_sum_heads(a[:, :1].contiguous())          # one KV head: the row itself
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert torch.equal(one, a[:, 0])
