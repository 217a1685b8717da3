"""Pins of the LaCache ladder oracle: ladder geometry, budgets, golden ladders, iteration."""

import os

import numpy as np
import pytest

from oracle import lacache as ol
from tests.test_oracle_kara import load_golden


def test_golden_ladders():
    cases = load_golden("lacache_ladders.txt")
    assert len(cases) == 4
    for c in cases:
        iv = {k: int(v[0]) for k, v in c.items() if not k.startswith("layer")}
        assert ol.check_params(iv["L"], iv["S"], iv["O"], iv["rung"], iv["budget"], iv["sink"],
                               iv["recent"])
        keep = ol.ladder_keep_slots(iv["n"], iv["L"], iv["S"], iv["O"], iv["rung"], iv["budget"],
                                    iv["sink"], iv["recent"])
        for layer in range(iv["L"]):
            assert keep[layer].tolist() == [int(x) for x in c[f"layer{layer}"]]


@pytest.mark.parametrize("L,S,O", [(32, 8, 4), (4, 2, 1), (8, 4, 2), (6, 3, 0), (12, 4, 2),
                                   (8, 8, 0), (8, 2, 0)])
def test_rung_spans_and_overlaps(L, S, O):
    stride = S - O
    for j in range(3 * L):
        layers = ol.rung_layers(j, L, S, O)
        assert len(set(layers)) == S
        first = layers[0]
        assert sorted(layers) == sorted((first + t) % L for t in range(S))    # cyclic run of S
        nxt = ol.rung_layers(j + 1, L, S, O)
        assert len(set(layers) & set(nxt)) == min(O, S) if S < L else True
        assert nxt[0] == (first + stride) % L


@pytest.mark.parametrize("L,S,O,rung,budget,sink,recent,extra", [
    (32, 8, 4, 64, 8192, 0, 0, 0), (32, 8, 4, 64, 8192, 0, 0, 12345), (4, 2, 1, 3, 24, 2, 4, 7),
    (8, 4, 2, 16, 96, 16, 16, 100), (6, 3, 0, 5, 40, 5, 5, 0), (8, 8, 0, 4, 64, 0, 0, 30)])
def test_every_layer_keeps_the_budget(L, S, O, rung, budget, sink, recent, extra):
    assert ol.check_params(L, S, O, rung, budget, sink, recent)
    n = ol.region_capacity(L, S, budget, sink, recent) + sink + recent + extra
    keep = ol.ladder_keep_slots(n, L, S, O, rung, budget, sink, recent)
    for k in keep:
        assert len(k) == budget and np.all(np.diff(k) > 0)
        assert k[:sink].tolist() == list(range(sink))
        assert k[len(k) - recent:].tolist() == list(range(n - recent, n))
    # every region slot that survives is kept in exactly S layers
    counts = np.zeros(n, dtype=int)
    for k in keep:
        counts[k] += 1
    region = counts[sink:n - recent]
    assert set(np.unique(region[region > 0]).tolist()) == {S}
    assert (region > 0).sum() == ol.region_capacity(L, S, budget, sink, recent)
    # the dropped slots are the oldest of the region
    kept_region = np.nonzero(region)[0]
    assert kept_region[0] == extra and kept_region[-1] == n - recent - sink - 1


def test_full_span_keeps_everything():
    keep = ol.ladder_keep_slots(64, 8, 8, 0, 4, 64)
    for k in keep:
        assert k.tolist() == list(range(64))


def test_invalid_params():
    assert not ol.check_params(8, 3, 1, 4, 64, 0, 0)     # stride 2 does not divide S = 3
    assert not ol.check_params(6, 4, 0, 4, 64, 0, 0)     # stride 4 does not divide L = 6
    assert not ol.check_params(8, 4, 4, 4, 64, 0, 0)     # O must be < S
    assert not ol.check_params(8, 4, 2, 4, 60, 0, 0)     # 60 is not a whole number of periods
    with pytest.raises(ValueError):
        ol.ladder_keep_slots(100, 8, 4, 2, 4, 64)        # not full: needs 128 region slots


def make_state(seed, page, bsz, n, layers, hkv, d, spare):
    rng = np.random.default_rng(seed)
    pages = -(-n // page)
    nb = bsz * pages + spare
    perm = rng.permutation(nb)
    table = np.full((bsz, pages + 1), -1, dtype=np.int32)
    for b in range(bsz):
        table[b, :pages] = perm[b * pages:(b + 1) * pages]
    free = np.zeros(nb, dtype=np.int32)
    free[:spare] = perm[bsz * pages:]
    ks = [rng.integers(0, 60000, size=(nb, page, hkv, d)).astype(np.uint16) for _ in range(layers)]
    vs = [rng.integers(0, 60000, size=(nb, page, hkv, d)).astype(np.uint16) for _ in range(layers)]
    ctx = np.full(bsz, n, dtype=np.int32)
    return ks, vs, table, ctx, free, spare


def test_lacache_compact_copies_and_conserves():
    page, L, S, O, rung, budget = 4, 4, 2, 1, 2, 8
    ks, vs, table, ctx, free, top = make_state(1, page, 2, 21, L, 2, 3, spare=6)
    st, kp, vp, bt, cl, fl, top2 = ol.lacache_compact(ks, vs, table, ctx, free, top, [0, 1], S, O,
                                                      rung, budget, 0, 0, page)
    assert st == ol.OK
    assert cl.tolist() == [budget, budget]
    used = set(int(x) for x in bt.ravel() if x >= 0)
    freed = set(int(x) for x in fl[:top2])
    assert not (used & freed) and len(used) + len(freed) == len(ks[0])
    for b in range(2):
        keep = ol.ladder_keep_slots(21, L, S, O, rung, budget)
        for layer in range(L):
            for t in range(budget):
                src = keep[layer][t]
                sb, sr = table[b, src // page], src % page
                db, dr = bt[b, t // page], t % page
                assert (kp[layer][db, dr] == ks[layer][sb, sr]).all()
                assert (vp[layer][db, dr] == vs[layer][sb, sr]).all()


def test_lacache_iteration_drops_oldest_first():
    # Pass 1 keeps slots of the newest R_max region; after appending, pass 2 sees the pass-1
    # survivors as its oldest slots and keeps fewer of them than of the new ones.
    L, S, O, rung, budget = 4, 2, 1, 1, 8
    r_max = ol.region_capacity(L, S, budget, 0, 0)      # 16
    keep1 = ol.ladder_keep_slots(40, L, S, O, rung, budget)
    assert min(k[0] for k in keep1) >= 40 - r_max
    n2 = budget + (r_max - budget)                       # refill to exactly R_max
    keep2 = ol.ladder_keep_slots(n2, L, S, O, rung, budget)
    old_kept = sum(int((k < budget).sum()) for k in keep2)
    new_kept = sum(int((k >= budget).sum()) for k in keep2)
    assert old_kept + new_kept == L * budget
    assert old_kept <= new_kept


def test_lacache_out_of_blocks_and_not_full():
    page = 4
    ks, vs, table, ctx, free, top = make_state(2, page, 1, 20, 4, 1, 2, spare=1)
    st, *_ = ol.lacache_compact(ks, vs, table, ctx, free, top, [0], 2, 1, 1, 8, 0, 0, page)
    assert st == ol.ERR_OUT_OF_BLOCKS
    st, *_ = ol.lacache_compact(ks, vs, table, ctx, free, top, [0], 2, 1, 1, 16, 0, 0, page)
    assert st == ol.ERR_INVALID_ARG
