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
    # W = 200: the fused kernel with a last CTA of 72 keys (mean and max)
    "w200": LAYER.with_(batch=3, ctx_lo=300, ctx_hi=700, window=200, keep=40),
    # more items than resident clusters: cluster ranges end inside items, the two parts are
    # added (mean) or maxed (max) by the split kernel
    "w256_split": synth.Workload("w256_split", batch=24, layers=1, hq=8, hkv=4, head_dim=128,
                                 ctx_lo=260, ctx_hi=420, window=256, keep=51, heavy_frac=0.05,
                                 spare_blocks=8),
    # head_dim 64: mean on the fused kernel, max on the two-pass kernels
    "d64_w256": synth.Workload("d64_w256", batch=3, layers=1, hq=8, hkv=2, head_dim=64,
                               ctx_lo=260, ctx_hi=400, window=256, keep=51, heavy_frac=0.05,
                               q_mode="neighbour", spare_blocks=8),
    # clusters of 16 CTAs (mean) and the two-pass kernels (max) at the largest fused window
    "w2048_fused": synth.Workload("w2048", batch=2, layers=1, hq=8, hkv=2, head_dim=128,
                                  ctx_lo=2050, ctx_hi=2600, window=2048, keep=409,
                                  heavy_frac=0.03, spare_blocks=8),
}
AGGS = {"mean": K.AGG_MEAN, "max": K.AGG_MAX}


def oracle_agg(cpu, wl, agg, rows=None):
    q = H.f64(cpu["q_win"][0])
    kf = H.f64(cpu["k"][0])
    bt, cl = H.i32(cpu["block_table"]), H.i32(cpu["ctx_len"])
    scale = 1 / math.sqrt(wl.head_dim)
    out = []
    for r in (range(wl.batch) if rows is None else rows):
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
    n0 = K.kara_launch_count()
    sc = K.kara_score_ex(dev["q_win"][0], dev["k"][0], pool, wl.window, agg=AGGS[agg],
                         status=status)
    torch.cuda.synchronize()
    launches = K.kara_launch_count() - n0
    assert K.read_status(status) == 0
    H.assert_scores_close(H.f64(sc), oracle_agg(cpu, wl, agg))
    # the fused kernel (and the split sum / max) for windows up to 1024 keys, and for the mean
    # at 2048; else the three two-pass kernels
    fused = ((wl.window <= 1024 and (agg == "mean" or wl.head_dim == 128))
             or (agg == "mean" and wl.window == 2048))
    assert (launches <= 2) == fused and (fused or launches == 3)
    if agg == "mean":   # the mean of each (sequence, KV head) row sums to 1
        assert np.allclose(H.f64(sc).sum(-1), 1.0, rtol=1e-4)


def test_max_skips_short_contexts_in_split_items():
    """The max aggregation with every third sequence too short for the window and cluster
    ranges ending inside items: those rows are zero and reported, the rest match the oracle."""
    wl = CASES["w256_split"]
    cpu, dev = H.make(wl, 4)
    bad = list(range(1, wl.batch, 3))
    good = [r for r in range(wl.batch) if r not in bad]
    dev["ctx_len"][bad] = wl.window - 1
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    sc = K.kara_score_ex(dev["q_win"][0], dev["k"][0], pool, wl.window, agg=K.AGG_MAX,
                         status=status)
    torch.cuda.synchronize()
    assert K.read_status(status) == K.ERR_INVALID_ARG
    assert (sc[bad] == 0).all()
    cpu["ctx_len"][bad] = wl.window - 1
    H.assert_scores_close(H.f64(sc[good]), oracle_agg(cpu, wl, "max", good))


def test_max_from_the_ring_equals_max_from_q_win():
    """The ring form reads the same query rows: the same tiles, the same result, bit for bit."""
    wl = CASES["w200"]
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


@pytest.mark.parametrize("name", ["w512_fused", "w2048_fused"])
def test_mean_from_the_ring_equals_mean_from_q_win_and_one_head_sums(name):
    wl = CASES[name]
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


# ---- the chunk-aware trim (kara_token2chunk_ex / kara_select_chunks_ex, KARA_TRIM_CHUNK) ----

def _golden(name):
    from tests.test_oracle_kara import load_golden
    return load_golden(name)


def test_chunk_trim_golden_cases_on_the_gpu():
    # the hand-worked cases through the kernels (fp32 scores keep the cases' orderings)
    for c in _golden("chunk_trim_cases.txt"):
        s = torch.tensor([c["scores"]], dtype=torch.float32, device="cuda")
        sel = torch.tensor([[int(x) for x in c["sel"]]], dtype=torch.int32, device="cuda")
        k = sel.shape[1]
        frac = int(c["num_anchors"][0]) / k
        args = (frac, int(c["gap_limit"][0]), int(c["widen"][0]))
        keep = K.kara_token2chunk(s, sel, *args, trim=K.TRIM_CHUNK)
        keep_tok = K.kara_token2chunk(s, sel, *args)
        keep_fused = K.kara_select_chunks(s, k, *args, trim=K.TRIM_CHUNK)
        torch.cuda.synchronize()
        assert H.i32(keep[0]).tolist() == [int(x) for x in c["keep"]]
        assert H.i32(keep_tok[0]).tolist() == [int(x) for x in c["keep_token"]]
        assert torch.equal(keep, keep_fused)


@pytest.mark.parametrize("seed", range(8))
def test_chunk_trim_matches_oracle(seed):
    # coarse scores (many ties, many short runs of U), random parameters, identical inputs on
    # both sides: identical keep sets; the fused kernel equals select then Token2Chunk
    rng = np.random.default_rng(100 + seed)
    rows, w = 6, int(rng.choice([64, 200, 1024, 2048]))
    k = int(rng.integers(1, max(2, w // 3)))
    s = (rng.integers(0, 7, size=(rows, w)).astype(np.float32) * 0.5
         + rng.random((rows, w)).astype(np.float32) * float(seed % 2))
    scores = torch.from_numpy(s).cuda()
    frac = float(np.float32(rng.choice([0.1, 0.25, 0.5, 1.0])))
    gap, wid = int(rng.integers(0, 10)), int(rng.integers(0, 3))
    sel = K.kara_select(scores, k)
    keep = K.kara_token2chunk(scores, sel, frac, gap, wid, trim=K.TRIM_CHUNK)
    sel2 = torch.empty_like(sel)
    keep2 = K.kara_select_chunks(scores, k, frac, gap, wid, sel=sel2, trim=K.TRIM_CHUNK)
    torch.cuda.synchronize()
    assert torch.equal(sel, sel2) and torch.equal(keep, keep2)
    s64 = s.astype(np.float64)
    na = ok.anchors_for(frac, k)
    for r in range(rows):
        ref = ok.token2chunk(s64[r], H.i32(sel[r]), na, gap, wid, trim="chunk")
        assert np.array_equal(H.i32(keep[r]), ref), r


def test_chunk_trim_on_window_scores_and_largest_window():
    # real window scores of the one-layer workload's shapes, and the largest window (4096 keys,
    # about 131 KB of shared memory with the chunk-aware trim's work arrays)
    wl = LAYER.with_(batch=2, ctx_lo=1100, ctx_hi=1400, window=1024, keep=204)
    cpu, dev = H.make(wl, 14)
    pool = K.PagedPool.from_cache(dev)
    sc = K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window)
    keep = K.kara_select_chunks(sc, wl.keep, wl.anchor_frac, wl.gap_limit, wl.widen,
                                trim=K.TRIM_CHUNK)
    rng = np.random.default_rng(3)
    big = torch.from_numpy(rng.random((2, 4096)).astype(np.float32)).cuda()
    keep_big = K.kara_select_chunks(big, 819, 0.25, 8, 1, trim=K.TRIM_CHUNK)
    torch.cuda.synchronize()
    s = H.f64(sc)
    na = ok.anchors_for(wl.anchor_frac, wl.keep)
    for r in range(wl.batch):
        for g in range(wl.hkv):
            ref = ok.token2chunk(s[r, g], ok.select_topk(s[r, g], wl.keep), na, wl.gap_limit,
                                 wl.widen, trim="chunk")
            assert np.array_equal(H.i32(keep[r, g]), ref)
    b64 = big.double().cpu().numpy()
    for r in range(2):
        ref = ok.token2chunk(b64[r], ok.select_topk(b64[r], 819), ok.anchors_for(0.25, 819), 8, 1,
                             trim="chunk")
        assert np.array_equal(H.i32(keep_big[r]), ref)
