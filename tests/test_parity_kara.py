"""GPU parity of the Kara path (score, select, Token2Chunk, compaction) against the oracle.

Scores: |gpu - oracle| <= 1e-3 |oracle| + 1e-6 (bf16 inputs, fp32 accumulation; the 1e-6 floor
covers terms the GPU's fp32 exponential flushes below 2^-126). Selection: identical sets given
identical scores; against oracle scores, sets equal except at near-ties (1e-3 relative).
Token2Chunk: identical given identical inputs. Compaction: bit-exact given the same keep.
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
SCORE_CASES = {
    "tiny": synth.WORKLOADS["tiny"],
    "g7_aligned": LAYER.with_(batch=3, ctx_lo=1024, ctx_hi=1024, window=256, keep=52),
    "g7_ragged_unaligned": LAYER.with_(batch=4, ctx_lo=300, ctx_hi=700, window=200, keep=40),
    "g7_w1024_unaligned": LAYER.with_(batch=2, ctx_lo=1030, ctx_hi=1400, window=1024, keep=204),
    "d64_g1": synth.Workload("d64_g1", batch=2, layers=1, hq=4, hkv=4, head_dim=64, ctx_lo=140,
                             ctx_hi=180, window=130, keep=26, heavy_frac=0.05, q_mode="neighbour",
                             spare_blocks=8),
    "g8_w384": synth.Workload("g8_w384", batch=2, layers=1, hq=16, hkv=2, head_dim=128,
                              ctx_lo=384, ctx_hi=500, window=384, keep=77, heavy_frac=0.03,
                              run_hi=16, q_mode="neighbour", spare_blocks=8),
    "w16_ctx_eq_w": synth.Workload("w16", batch=3, layers=1, hq=2, hkv=1, head_dim=128,
                                   ctx_lo=16, ctx_hi=16, window=16, keep=1, spare_blocks=4),
    # windows of 128 * c keys take the fused cluster kernel (c CTAs per cluster)
    "g7_w512_ragged": LAYER.with_(batch=4, ctx_lo=520, ctx_hi=900, window=512, keep=102),
    "d64_g4_w256": synth.Workload("d64_g4_w256", batch=3, layers=1, hq=8, hkv=2, head_dim=64,
                                  ctx_lo=260, ctx_hi=400, window=256, keep=51, heavy_frac=0.05,
                                  q_mode="neighbour", spare_blocks=8),
    # more (sequence, KV head) items than resident clusters: cluster ranges end inside items,
    # whose two parts are summed by the split kernel
    "w128_split_items": synth.Workload("w128_split", batch=40, layers=1, hq=8, hkv=4,
                                       head_dim=128, ctx_lo=130, ctx_hi=300, window=128, keep=26,
                                       heavy_frac=0.05, q_mode="neighbour", spare_blocks=8),
    "w256_split_items": synth.Workload("w256_split", batch=24, layers=1, hq=8, hkv=4,
                                       head_dim=128, ctx_lo=260, ctx_hi=420, window=256, keep=51,
                                       heavy_frac=0.05, spare_blocks=8),
    # W = 1024 on clusters of 8: 18 items over the resident clusters, ranges end inside items
    # (the bench's instantiation of the split-item sum, every row element-checked); and 12
    # ragged rows of 2 query heads per KV head
    "w1024_split_items": synth.Workload("w1024_split", batch=9, layers=1, hq=2, hkv=2,
                                        head_dim=128, ctx_lo=1030, ctx_hi=1500, window=1024,
                                        keep=204, heavy_frac=0.05, q_mode="neighbour",
                                        spare_blocks=8),
    # 332 (row, KV head) items at W = 1024: the clusters fill the GPU, and the last 28 items
    # go to the one-CTA-per-item two-pass helper on the SMs the clusters leave idle
    "w1024_helper": synth.Workload("w1024_helper", batch=83, layers=1, hq=4, hkv=4,
                                   head_dim=128, ctx_lo=1030, ctx_hi=1200, window=1024,
                                   keep=204, heavy_frac=0.05, q_mode="neighbour",
                                   spare_blocks=8),
    "w1024_g2": synth.Workload("w1024_g2", batch=12, layers=1, hq=8, hkv=4,
                                   head_dim=128, ctx_lo=1024, ctx_hi=1800, window=1024,
                                   keep=204, heavy_frac=0.05, spare_blocks=8),
    # windows that are not a multiple of 128: the last CTA of the cluster owns fewer keys
    # (W = 1000 on 8 CTAs, the last with 104); windows between 1024 and 2048 and above 2048
    # (up to the largest, 4096) take the two-pass kernels
    "w1000_partial": synth.Workload("w1000", batch=3, layers=1, hq=8, hkv=2, head_dim=128,
                                    ctx_lo=1000, ctx_hi=1400, window=1000, keep=200,
                                    heavy_frac=0.05, q_mode="neighbour", spare_blocks=8),
    "w1100_twopass": synth.Workload("w1100", batch=3, layers=1, hq=4, hkv=2, head_dim=128,
                                 ctx_lo=1100, ctx_hi=1500, window=1100, keep=220,
                                 heavy_frac=0.05, spare_blocks=8),
    "w4096_largest": synth.Workload("w4096", batch=1, layers=1, hq=2, hkv=1, head_dim=128,
                                    ctx_lo=4100, ctx_hi=4200, window=4096, keep=819,
                                    heavy_frac=0.03, spare_blocks=8),
    "w2500_twopass": synth.Workload("w2500", batch=2, layers=1, hq=4, hkv=2, head_dim=128,
                                    ctx_lo=2500, ctx_hi=2900, window=2500, keep=500,
                                    heavy_frac=0.03, spare_blocks=8),
    # W = 2048: clusters of 16 CTAs (non-portable size); whole items per cluster, then more
    # items than resident clusters of 16 (at most 148 / 16 of them)
    "g4_w2048_ragged": synth.Workload("g4_w2048", batch=3, layers=1, hq=8, hkv=2, head_dim=128,
                                      ctx_lo=2050, ctx_hi=2900, window=2048, keep=409,
                                      heavy_frac=0.03, run_hi=16, spare_blocks=8),
    "w2048_split_items": synth.Workload("w2048_split", batch=8, layers=1, hq=4, hkv=2,
                                        head_dim=128, ctx_lo=2048, ctx_hi=2400, window=2048,
                                        keep=409, heavy_frac=0.05, q_mode="neighbour",
                                        spare_blocks=8),
}


def oracle_scores(cpu, wl, seq_ids=None):
    """Oracle scores of the due rows `seq_ids` (default: every row in order); the window
    queries of due row i are those of sequence seq_ids[i]."""
    q = H.f64(cpu["q_win"][0])
    if seq_ids is None:
        seq_ids = list(range(wl.batch))
    else:
        q = q[seq_ids]
    return ok.score_batch(q, H.f64(cpu["k"][0]), H.i32(cpu["block_table"]), H.i32(cpu["ctx_len"]),
                          seq_ids, wl.window, 1 / math.sqrt(wl.head_dim), wl.page)


@pytest.mark.parametrize("name", list(SCORE_CASES))
def test_score_matches_oracle(name):
    wl = SCORE_CASES[name]
    cpu, dev = H.make(wl, 11)
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    scores = K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window, status=status)
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    ref = oracle_scores(cpu, wl)
    H.assert_scores_close(H.f64(scores), ref)
    # invariant at any size: every row of scores sums to W * G
    sums = scores.double().sum(-1).cpu().numpy()
    assert np.allclose(sums, wl.window * wl.group, rtol=1e-4)


@pytest.mark.parametrize("name,ids", [("g7_ragged_unaligned", [1, 3]), ("g7_w512_ragged", [1, 3]),
                                      ("w1024_g2", [7, 0, 11, 3, 9, 1, 5, 10, 2, 8, 4, 6]),
                                      ("w1024_helper", list(range(82, -1, -1)))])
def test_score_subset_of_sequences(name, ids):
    """Due rows given by seq_ids: a subset, or every row in another order (with the helper's
    rows looked up through seq_ids too)."""
    wl = SCORE_CASES[name]
    cpu, dev = H.make(wl, 5)
    assert wl.batch > max(ids)
    pool = K.PagedPool.from_cache(dev)
    q = dev["q_win"][0][ids].contiguous()
    seq = torch.tensor(ids, dtype=torch.int32, device="cuda")
    scores = K.kara_score(q, dev["k"][0], pool, wl.window, seq_ids=seq)
    torch.cuda.synchronize()
    H.assert_scores_close(H.f64(scores), oracle_scores(cpu, wl, ids))


def test_score_reports_short_context():
    wl = SCORE_CASES["g7_aligned"]
    cpu, dev = H.make(wl, 2)
    dev["ctx_len"][1] = wl.window - 1
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    scores = K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window, status=status)
    torch.cuda.synchronize()
    assert K.read_status(status) == K.ERR_INVALID_ARG
    assert (scores[1] == 0).all()
    cpu["ctx_len"][1] = wl.window - 1
    ref = oracle_scores(cpu, wl, [0, 2])
    H.assert_scores_close(H.f64(scores[[0, 2]]), ref)


def test_score_w2048_helper_rows():
    """W = 2048 with items enough for the helper beside clusters of 16 (65 rows of 4 KV heads:
    the last 36 items, rows 56-64, on the idle SMs): the helper's rows and a few of the fused
    kernel's against the oracle, every row's sum W * G."""
    wl = synth.Workload("w2048_helper", batch=65, layers=1, hq=4, hkv=4, head_dim=128,
                        ctx_lo=2050, ctx_hi=2200, window=2048, keep=409, heavy_frac=0.03,
                        spare_blocks=8)
    cpu, dev = H.make(wl, 9)
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    c0 = K.kara_launch_count()
    scores = K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window, status=status)
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    assert K.kara_launch_count() - c0 in (1, 2, 3)
    sums = scores.double().sum(-1).cpu().numpy()
    assert np.allclose(sums, wl.window * wl.group, rtol=1e-4)
    rows = [0, 1, 30] + list(range(wl.batch - 10, wl.batch))
    H.assert_scores_close(H.f64(scores[rows]), oracle_scores(cpu, wl, rows))


def test_score_ring_equals_dense_with_the_helper():
    """The window-query ring form with the helper active (83 due rows at W = 1024, seq_ids
    given): the same tiles in the same order as the dense form, so the same bits."""
    wl = SCORE_CASES["w1024_helper"]
    cpu, dev = H.make(wl, 10)
    pool = K.PagedPool.from_cache(dev)
    W = wl.window
    ring = torch.zeros((wl.batch, 2 * W, wl.hq, wl.head_dim), device="cuda", dtype=torch.bfloat16)
    for b in range(wl.batch):
        off = (int(cpu["ctx_len"][b]) - W) % W
        ring[b, off:off + W] = dev["q_win"][0][b]
    seq = torch.arange(wl.batch, dtype=torch.int32, device="cuda")
    a = K.kara_score(dev["q_win"][0], dev["k"][0], pool, W)
    b = K.kara_score_ex(ring, dev["k"][0], pool, W, ring=True, seq_ids=seq)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_score_helper_rows_report_short_contexts():
    """Too-short contexts among the helper's rows and the fused kernel's: their rows are zero
    and reported, the rest match the oracle."""
    wl = SCORE_CASES["w1024_helper"]
    cpu, dev = H.make(wl, 7)
    bad = [wl.batch - 1, wl.batch - 4, 3]
    good = [r for r in range(wl.batch) if r not in bad]
    dev["ctx_len"][bad] = wl.window - 1
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    scores = K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window, status=status)
    torch.cuda.synchronize()
    assert K.read_status(status) == K.ERR_INVALID_ARG
    assert (scores[bad] == 0).all()
    cpu["ctx_len"][bad] = wl.window - 1
    H.assert_scores_close(H.f64(scores[good]), oracle_scores(cpu, wl, good))


def test_score_w1024_reports_short_contexts():
    """Too-short contexts among the rows of a W=1024 launch (the last row and one inside):
    their rows are zero and reported, the rest match the oracle."""
    wl = SCORE_CASES["w1024_g2"]
    cpu, dev = H.make(wl, 6)
    bad = [wl.batch - 1, 2]
    good = [r for r in range(wl.batch) if r not in bad]
    dev["ctx_len"][bad] = wl.window - 1
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    scores = K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window, status=status)
    torch.cuda.synchronize()
    assert K.read_status(status) == K.ERR_INVALID_ARG
    assert (scores[bad] == 0).all()
    cpu["ctx_len"][bad] = wl.window - 1
    H.assert_scores_close(H.f64(scores[good]), oracle_scores(cpu, wl, good))


def test_score_split_items_skip_short_contexts():
    """Every third sequence too short for the window: its items drop out of the cluster ranges
    (and of the split sums), its rows are zero and reported; the rest match the oracle."""
    wl = SCORE_CASES["w128_split_items"]
    cpu, dev = H.make(wl, 4)
    bad = list(range(1, wl.batch, 3))
    good = [r for r in range(wl.batch) if r not in bad]
    dev["ctx_len"][bad] = wl.window - 1
    pool = K.PagedPool.from_cache(dev)
    status = K.new_status()
    scores = K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window, status=status)
    torch.cuda.synchronize()
    assert K.read_status(status) == K.ERR_INVALID_ARG
    assert (scores[bad] == 0).all()
    cpu["ctx_len"][bad] = wl.window - 1
    H.assert_scores_close(H.f64(scores[good]), oracle_scores(cpu, wl, good))


@pytest.mark.parametrize("name,launches", [("g7_w1024_unaligned", (1,)), ("w128_split_items", (2,)),
                                           ("w1024_split_items", (2,)), ("w1024_helper", (2, 3)),
                                           ("g7_ragged_unaligned", (1, 2)), ("w1100_twopass", (3,)),
                                           ("w2500_twopass", (3,)),
                                           ("g4_w2048_ragged", (1,)), ("w2048_split_items", (2,))])
def test_score_launch_count(name, launches):
    """The fused kernel alone when every cluster range holds whole items; with the split sum
    when more items than resident clusters make ranges end inside items; with the one-kernel
    helper when the clusters fill the GPU and there are items enough for it; three two-pass
    kernels above W = 2048."""
    wl = SCORE_CASES[name]
    cpu, dev = H.make(wl, 1)
    pool = K.PagedPool.from_cache(dev)
    c0 = K.kara_launch_count()
    K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window)
    torch.cuda.synchronize()
    assert K.kara_launch_count() - c0 in launches


@pytest.mark.parametrize("name", ["tiny", "g7_ragged_unaligned", "g8_w384", "w16_ctx_eq_w"])
def test_select_and_token2chunk(name):
    wl = SCORE_CASES[name]
    cpu, dev = H.make(wl, 21)
    pool = K.PagedPool.from_cache(dev)
    scores = K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window)
    sel = K.kara_select(scores, wl.keep)
    na = wl.anchor_frac
    keep = K.kara_token2chunk(scores, sel, na, wl.gap_limit, wl.widen)
    torch.cuda.synchronize()
    s_gpu = H.f64(scores)
    # identical inputs -> identical outputs
    assert np.array_equal(H.i32(sel), ok.select_batch(s_gpu, wl.keep))
    assert np.array_equal(H.i32(keep), ok.token2chunk_batch(s_gpu, H.i32(sel),
                                                            ok.anchors_for(na, wl.keep),
                                                            wl.gap_limit, wl.widen))
    # against the oracle's own scores: equal up to near-ties
    ref = oracle_scores(cpu, wl)
    H.assert_selection_matches(H.i32(sel), ok.select_batch(ref, wl.keep), ref)


@pytest.mark.parametrize("seed", range(6))
def test_select_ties_and_token2chunk_params(seed):
    rng = np.random.default_rng(seed)
    rows, w = 7, int(rng.integers(16, 2049))
    k = int(rng.integers(1, w + 1))
    # coarse values force many exact ties; include -0.0 and +0.0
    s = rng.integers(0, 5, size=(rows, w)).astype(np.float32) * 0.25
    s[0, :8] = -0.0
    scores = torch.from_numpy(s).cuda()
    sel = K.kara_select(scores, k)
    # an anchor fraction in single precision, as the C ABI takes it; the oracle gets the same
    # value (ceil of the product rounded to 6 decimals on both sides)
    frac = float(np.float32(rng.choice([0.0, 0.1, 0.2, 0.25, 0.5, 0.75, 1.0, rng.random()])))
    gap = int(rng.integers(0, 12))
    wid = int(rng.integers(0, 4))
    keep = K.kara_token2chunk(scores, sel, frac, gap, wid)
    torch.cuda.synchronize()
    assert np.array_equal(H.i32(sel), ok.select_batch(s.astype(np.float64), k))
    assert np.array_equal(H.i32(keep), ok.token2chunk_batch(s.astype(np.float64), H.i32(sel),
                                                            ok.anchors_for(frac, k), gap, wid))


@pytest.mark.parametrize("frac,k,count", [(0.0, 61, 0), (0.5, 61, 31), (1.0, 61, 61),
                                          (0.2, 61, 13), (0.2, 5, 1)])
def test_anchor_fraction_through_the_c_abi(frac, k, count):
    # the C ABI takes anchor_frac and counts ceil(frac * k) anchors itself (0.2 arrives as the
    # float 0.2000000030, still one anchor of five)
    assert ok.anchors_for(frac, k) == count
    rng = np.random.default_rng(11)
    s = rng.random((4, 300)).astype(np.float32)
    scores = torch.from_numpy(s).cuda()
    sel = K.kara_select(scores, k)
    keep = K.kara_token2chunk(scores, sel, frac, 8, 1)
    keep2 = K.kara_select_chunks(scores, k, frac, 8, 1)
    torch.cuda.synchronize()
    assert torch.equal(keep, keep2)
    s64 = s.astype(np.float64)
    for r in range(4):
        ref = ok.token2chunk(s64[r], ok.select_topk(s64[r], k), count, 8, 1)
        assert np.array_equal(H.i32(keep[r]), ref)


def test_select_max_window_and_k_equals_w():
    rng = np.random.default_rng(3)
    s = rng.random((3, 4096)).astype(np.float32)
    scores = torch.from_numpy(s).cuda()
    for k in (1, 819, 4096):
        sel = K.kara_select(scores, k)
        torch.cuda.synchronize()
        assert np.array_equal(H.i32(sel), ok.select_batch(s.astype(np.float64), k))
    # Token2Chunk at the largest window (58 KB of shared memory), separately and fused
    sel = K.kara_select(scores, 819)
    keep = K.kara_token2chunk(scores, sel, 0.5, 8, 1)          # ceil(0.5 * 819) = 410 anchors
    keep2 = K.kara_select_chunks(scores, 819, 0.5, 8, 1)
    torch.cuda.synchronize()
    assert torch.equal(keep, keep2)
    s64 = s.astype(np.float64)
    for r in range(3):
        assert np.array_equal(H.i32(keep[r]), ok.token2chunk(s64[r], ok.select_topk(s64[r], 819),
                                                            410, 8, 1))


# ---------------------------------------------------------------- compaction

def oracle_compact(cpu, wl, keep, seq_ids, layers):
    return ok.compact([H.bits(cpu["k"][i]) for i in range(layers)],
                      [H.bits(cpu["v"][i]) for i in range(layers)],
                      H.i32(cpu["block_table"]), H.i32(cpu["ctx_len"]), H.i32(cpu["free_list"]),
                      int(cpu["free_top"][0]), seq_ids, wl.window, keep, wl.page)


def check_compaction(dev, ref, layers, seq_ids, batch):
    st, kp, vp, bt, cl, fl, top, fresh = ref
    assert st == ok.OK
    assert np.array_equal(H.i32(dev["block_table"]), bt)
    assert np.array_equal(H.i32(dev["ctx_len"]), cl)
    assert int(dev["free_top"][0]) == top
    assert np.array_equal(H.i32(dev["free_list"])[:top], fl[:top])
    for layer in range(layers):
        kg, vg = H.bits(dev["k"][layer]), H.bits(dev["v"][layer])
        for b in range(batch):
            n = int(cl[b])
            assert np.array_equal(H.logical_rows(kg, bt[b], n), H.logical_rows(kp[layer], bt[b], n))
            assert np.array_equal(H.logical_rows(vg, bt[b], n), H.logical_rows(vp[layer], bt[b], n))
        touched = set(x for ids in fresh.values() for x in ids)
        untouched = np.array(sorted(set(range(kg.shape[0])) - touched))
        assert np.array_equal(kg[untouched], kp[layer][untouched])
        assert np.array_equal(vg[untouched], vp[layer][untouched])


@pytest.mark.parametrize("name,layers,subset", [("tiny", 1, None), ("g7_ragged_unaligned", 3, None),
                                                ("g7_ragged_unaligned", 2, [0, 2, 3]),
                                                ("d64_g1", 2, [1]), ("w16_ctx_eq_w", 1, None)])
def test_compact_bit_exact(name, layers, subset):
    wl = SCORE_CASES[name]
    cpu, dev = H.make(wl, 31, layers=layers)
    seq_ids = list(range(wl.batch)) if subset is None else subset
    rng = np.random.default_rng(9)
    keep = np.stack([synth.random_keep(rng, len(seq_ids) * wl.hkv, wl.window, wl.keep)
                     .reshape(len(seq_ids), wl.hkv, wl.keep) for _ in range(layers)])
    ref = oracle_compact(cpu, wl, keep, seq_ids, layers)
    pool = K.PagedPool.from_cache(dev)
    sid = None if subset is None else torch.tensor(subset, dtype=torch.int32, device="cuda")
    status = K.kara_compact(dev["k"], dev["v"], pool, wl.window,
                            torch.from_numpy(keep).cuda(), seq_ids=sid)
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    check_compaction(dev, ref, layers, seq_ids, wl.batch)


def test_compact_keep_all_window():
    wl = SCORE_CASES["g7_ragged_unaligned"].with_(keep=200)
    cpu, dev = H.make(wl, 8)
    keep = np.tile(np.arange(wl.window, dtype=np.int32), (1, wl.batch, wl.hkv, 1))
    ref = oracle_compact(cpu, wl, keep, list(range(wl.batch)), 1)
    pool = K.PagedPool.from_cache(dev)
    K.kara_compact(dev["k"], dev["v"], pool, wl.window, torch.from_numpy(keep).cuda())
    torch.cuda.synchronize()
    check_compaction(dev, ref, 1, list(range(wl.batch)), wl.batch)


def test_compact_out_of_blocks_changes_nothing():
    wl = SCORE_CASES["g7_ragged_unaligned"]
    cpu, dev = H.make(wl, 4)
    dev["free_top"][0] = 2
    before = {k: dev[k].clone() for k in ("block_table", "ctx_len", "free_list", "free_top")}
    kb = dev["k"][0].clone()
    keep = np.tile(np.arange(wl.keep, dtype=np.int32), (1, wl.batch, wl.hkv, 1))
    pool = K.PagedPool.from_cache(dev)
    status = K.kara_compact(dev["k"], dev["v"], pool, wl.window, torch.from_numpy(keep).cuda())
    torch.cuda.synchronize()
    assert K.read_status(status) == K.ERR_OUT_OF_BLOCKS
    for k, t in before.items():
        assert torch.equal(dev[k], t)
    assert torch.equal(dev["k"][0], kb)


@pytest.mark.parametrize("bad", ["past_window", "negative", "out_of_order"])
def test_compact_bad_keep_changes_nothing(bad):
    # one bad entry in the last layer's last row: the whole call is refused before anything
    # moves (the check runs before the plan pops or frees a block)
    wl = SCORE_CASES["g7_ragged_unaligned"]
    cpu, dev = H.make(wl, 5, layers=2)
    rng = np.random.default_rng(3)
    keep = np.stack([synth.random_keep(rng, wl.batch * wl.hkv, wl.window, wl.keep)
                     .reshape(wl.batch, wl.hkv, wl.keep) for _ in range(2)])
    if bad == "past_window":
        keep[1, -1, -1, -1] = wl.window
    elif bad == "negative":
        keep[1, -1, -1, 0] = -1
    else:
        keep[1, -1, -1, [3, 4]] = keep[1, -1, -1, [4, 3]]
    st_ref = oracle_compact(cpu, wl, keep, list(range(wl.batch)), 2)[0]
    assert st_ref == ok.ERR_INVALID_ARG
    before = {k: dev[k].clone() for k in ("block_table", "ctx_len", "free_list", "free_top")}
    pools = [t.clone() for t in dev["k"] + dev["v"]]
    pool = K.PagedPool.from_cache(dev)
    status = K.kara_compact(dev["k"], dev["v"], pool, wl.window, torch.from_numpy(keep).cuda())
    torch.cuda.synchronize()
    assert K.read_status(status) == K.ERR_INVALID_ARG
    for k, t in before.items():
        assert torch.equal(dev[k], t), k
    for t, t0 in zip(dev["k"] + dev["v"], pools):
        assert torch.equal(t, t0)


def test_compact_bad_block_id_is_reported_not_faulted():
    wl = SCORE_CASES["g7_ragged_unaligned"]
    cpu, dev = H.make(wl, 4)
    n = int(cpu["ctx_len"][1])
    dev["block_table"][1, (n - 1) // 16] = 10 ** 8
    keep = np.tile(np.arange(wl.keep, dtype=np.int32), (1, wl.batch, wl.hkv, 1))
    pool = K.PagedPool.from_cache(dev)
    status = K.kara_compact(dev["k"], dev["v"], pool, wl.window, torch.from_numpy(keep).cuda())
    scores_status = K.new_status()
    K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window, status=scores_status)
    torch.cuda.synchronize()
    assert K.read_status(status) == K.ERR_BAD_BLOCK
    assert K.read_status(scores_status) == K.ERR_BAD_BLOCK


def test_compact_reuses_freed_blocks():
    # A second compaction, after appending W tokens to each sequence, pops blocks the first
    # one freed (block free and reuse).
    wl = SCORE_CASES["g7_ragged_unaligned"].with_(spare_blocks=32)
    cpu, dev = H.make(wl, 17)
    rng = np.random.default_rng(2)
    keep1 = synth.random_keep(rng, wl.batch * wl.hkv, wl.window, wl.keep).reshape(
        1, wl.batch, wl.hkv, wl.keep)
    ref1 = oracle_compact(cpu, wl, keep1, list(range(wl.batch)), 1)
    pool = K.PagedPool.from_cache(dev)
    K.kara_compact(dev["k"], dev["v"], pool, wl.window, torch.from_numpy(keep1).cuda())
    torch.cuda.synchronize()
    check_compaction(dev, ref1, 1, list(range(wl.batch)), wl.batch)
    _, kp, vp, bt, cl, fl, top, fresh1 = ref1
    old_table = H.i32(cpu["block_table"])
    freed1 = set(old_table[old_table >= 0].tolist()) - set(bt[bt >= 0].tolist())
    assert freed1 and freed1 <= set(fl[:top].tolist())
    # append W slots per sequence on the host state, taking blocks from the free list top
    # (the table gets room for the longer sequences)
    bt = np.pad(bt, ((0, 0), (0, wl.window // 16 + 2)), constant_values=-1)
    cl, fl = cl.copy(), fl.copy()
    for b in range(wl.batch):
        n = int(cl[b])
        for p in range(n // 16 + (1 if n % 16 else 0), (n + wl.window + 15) // 16):
            top -= 1
            bt[b, p] = fl[top]
        cl[b] = n + wl.window
    cpu2 = dict(cpu)
    cpu2["k"] = [torch.from_numpy(kp[0]).view(torch.bfloat16)]
    cpu2["v"] = [torch.from_numpy(vp[0]).view(torch.bfloat16)]
    cpu2["block_table"] = torch.from_numpy(bt.astype(np.int32))
    cpu2["ctx_len"] = torch.from_numpy(cl.astype(np.int32))
    cpu2["free_list"] = torch.from_numpy(fl.astype(np.int32))
    cpu2["free_top"] = torch.tensor([top], dtype=torch.int32)
    dev2 = H.to_device(cpu2)
    keep2 = synth.random_keep(rng, wl.batch * wl.hkv, wl.window, wl.keep).reshape(
        1, wl.batch, wl.hkv, wl.keep)
    ref2 = oracle_compact(cpu2, wl, keep2, list(range(wl.batch)), 1)
    pool2 = K.PagedPool.from_cache(dev2)
    K.kara_compact(dev2["k"], dev2["v"], pool2, wl.window, torch.from_numpy(keep2).cuda())
    torch.cuda.synchronize()
    check_compaction(dev2, ref2, 1, list(range(wl.batch)), wl.batch)
    used2 = set(x for ids in ref2[7].values() for x in ids) | set(bt[bt >= 0].ravel().tolist())
    assert used2 & freed1, "the second pass should reuse blocks the first one freed"


@pytest.mark.parametrize("name", ["g7_ragged_unaligned", "g8_w384", "w16_ctx_eq_w"])
def test_select_chunks_equals_select_then_token2chunk(name):
    """The fused select + Token2Chunk kernel gives the separate calls' keep (and selection)
    bit for bit, and both equal the oracle's on the same scores."""
    wl = SCORE_CASES[name]
    cpu, dev = H.make(wl, 12)
    pool = K.PagedPool.from_cache(dev)
    sc = K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window)
    na = wl.anchor_frac
    sel = K.kara_select(sc, wl.keep)
    keep = K.kara_token2chunk(sc, sel, na, wl.gap_limit, wl.widen)
    sel2 = torch.empty_like(sel)
    keep2 = K.kara_select_chunks(sc, wl.keep, na, wl.gap_limit, wl.widen, sel=sel2)
    keep3 = K.kara_select_chunks(sc, wl.keep, na, wl.gap_limit, wl.widen)
    torch.cuda.synchronize()
    assert torch.equal(keep, keep2) and torch.equal(sel, sel2) and torch.equal(keep, keep3)
    s = H.f64(sc)
    for r in range(wl.batch):
        for g in range(wl.hkv):
            ref = ok.token2chunk(s[r, g], ok.select_topk(s[r, g], wl.keep),
                                 ok.anchors_for(na, wl.keep), wl.gap_limit, wl.widen)
            assert np.array_equal(H.i32(keep2[r, g]), ref)


@pytest.mark.parametrize("name,layers,subset", [("g7_ragged_unaligned", 2, False),
                                                ("g7_w512_ragged", 1, True),
                                                ("d64_g4_w256", 3, False)])
def test_compress_equals_select_chunks_then_compact(name, layers, subset):
    """kara_compress (plan, then selection + Token2Chunk + gather in one kernel per row) leaves
    the same cache, table, lengths, free list and keep sets as kara_select_chunks on every
    layer followed by kara_compact, bit for bit; both against the oracle."""
    wl = SCORE_CASES[name].with_(layers=layers)
    cpu, dev_a = H.make(wl, 15)
    dev_b = H.to_device(cpu)
    ids = [1, 3] if subset else list(range(wl.batch))
    assert wl.batch > max(ids)
    seq = torch.tensor(ids, dtype=torch.int32, device="cuda")
    na = wl.anchor_frac
    pool_a, pool_b = K.PagedPool.from_cache(dev_a), K.PagedPool.from_cache(dev_b)
    scores = torch.stack([K.kara_score(dev_a["q_win"][l][ids].contiguous(), dev_a["k"][l], pool_a,
                                       wl.window, seq_ids=seq) for l in range(layers)])
    keep_a = torch.empty((layers, len(ids), wl.hkv, wl.keep), dtype=torch.int32, device="cuda")
    for l in range(layers):
        K.kara_select_chunks(scores[l], wl.keep, na, wl.gap_limit, wl.widen, keep=keep_a[l])
    st_a = K.kara_compact(dev_a["k"], dev_a["v"], pool_a, wl.window, keep_a, seq_ids=seq)
    keep_b = torch.empty_like(keep_a)
    st_b = K.kara_compress(scores, dev_b["k"], dev_b["v"], pool_b, wl.window, wl.keep, na,
                           wl.gap_limit, wl.widen, seq_ids=seq, keep=keep_b)
    torch.cuda.synchronize()
    assert K.read_status(st_a) == 0 and K.read_status(st_b) == 0
    assert torch.equal(keep_a, keep_b)
    for key in ("block_table", "ctx_len", "free_top"):
        assert torch.equal(dev_a[key], dev_b[key])
    top = int(dev_a["free_top"][0])
    assert torch.equal(dev_a["free_list"][:top], dev_b["free_list"][:top])
    bt, cl = H.i32(dev_a["block_table"]), H.i32(dev_a["ctx_len"])
    for l in range(layers):
        ka, kb = H.bits(dev_a["k"][l]), H.bits(dev_b["k"][l])
        va, vb = H.bits(dev_a["v"][l]), H.bits(dev_b["v"][l])
        for b in range(wl.batch):
            n = int(cl[b])
            assert np.array_equal(H.logical_rows(ka, bt[b], n), H.logical_rows(kb, bt[b], n))
            assert np.array_equal(H.logical_rows(va, bt[b], n), H.logical_rows(vb, bt[b], n))
    # and the oracle's compaction with those keep sets
    check_compaction(dev_b, oracle_compact(cpu, wl, H.i32(keep_b), ids, layers), layers, ids,
                     wl.batch)


def test_compress_out_of_blocks_changes_nothing():
    wl = SCORE_CASES["g7_ragged_unaligned"]
    cpu, dev = H.make(wl, 16)
    dev["free_top"].fill_(1)
    pool = K.PagedPool.from_cache(dev)
    before = {k2: dev[k2].clone() for k2 in ("block_table", "ctx_len", "free_top")}
    kb = H.bits(dev["k"][0]).copy()
    scores = K.kara_score(dev["q_win"][0], dev["k"][0], pool, wl.window)[None]
    na = wl.anchor_frac
    st = K.kara_compress(scores, dev["k"], dev["v"], pool, wl.window, wl.keep, na, wl.gap_limit,
                         wl.widen)
    torch.cuda.synchronize()
    assert K.read_status(st) == K.ERR_OUT_OF_BLOCKS
    for k2, t in before.items():
        assert torch.equal(dev[k2], t)
    assert np.array_equal(H.bits(dev["k"][0]), kb)
