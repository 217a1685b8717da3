"""The seeded generators: determinism, block bookkeeping, heavy-run coverage, query recipe."""

import numpy as np
import torch

from decode_kv_cache_kara_b200 import synth


def test_tiny_cache_is_deterministic_and_consistent():
    wl = synth.WORKLOADS["tiny"]
    a = synth.make_cache(wl, 1234)
    b = synth.make_cache(wl, 1234)
    assert torch.equal(a["k"][0], b["k"][0]) and torch.equal(a["q_win"][0], b["q_win"][0])
    table = a["block_table"].numpy()
    top = int(a["free_top"][0])
    used = table[table >= 0]
    free = a["free_list"].numpy()[:top]
    assert len(set(used.tolist()) | set(free.tolist())) == a["num_blocks"]
    assert not (set(used.tolist()) & set(free.tolist()))
    assert a["q_win"][0].shape == (1, 128, 4, 64)


def test_heavy_runs_cover_the_target_fraction():
    wl = synth.WORKLOADS["tiny"].with_(heavy_scale=4.0)
    c = synth.make_cache(wl, 7)
    n = int(c["ctx_len"][0])
    slots = np.arange(n)
    tab = c["block_table"][0].numpy()
    k = c["k"][0][tab[slots // 16], slots % 16].float()          # [n, Hkv, d]
    norms = k.norm(dim=-1).mean(dim=-1)
    heavy = (norms > 2.5 * np.sqrt(64)).numpy()
    assert not heavy[: n - wl.window].any()                        # window-only heavy keys
    assert abs(heavy.sum() - round(0.05 * wl.window)) <= wl.run_hi


def test_neighbour_queries_follow_previous_key():
    wl = synth.WORKLOADS["layer"].with_(batch=2, ctx_lo=160, ctx_hi=300, window=64, keep=12)
    c = synth.make_cache(wl, 3)
    q = c["q_win"][0].float()
    for b in range(2):
        n = int(c["ctx_len"][b])
        s = n - wl.window + 5 - 1
        blk = int(c["block_table"][b, s // 16])
        kprev = c["k"][0][blk, s % 16].float()                     # [Hkv, d]
        diff = q[b, 5] - kprev.repeat_interleave(wl.group, 0)
        assert 0.3 < float(diff.std()) < 0.7


def test_decode_step_inputs_are_seeded_and_shaped():
    wl = synth.Workload("s", batch=3, layers=2, hq=8, hkv=2, head_dim=64, ctx_lo=20, ctx_hi=40,
                        window=16, keep=4)
    a = synth.decode_step_inputs(wl, 7, 3)
    b = synth.decode_step_inputs(wl, 7, 3)
    c = synth.decode_step_inputs(wl, 7, 4)
    assert len(a) == wl.layers
    for la, lb, lc in zip(a, b, c):
        assert la["q"].shape == (3, 8, 64) and la["k"].shape == (3, 2, 64)
        assert all(x.dtype == torch.bfloat16 for x in la.values())
        assert all(torch.equal(la[n], lb[n]) for n in la)          # same (seed, step)
        assert not torch.equal(la["k"], lc["k"])                   # another step differs
    # each query head is its KV head's new key plus noise of scale 0.5
    d = (a[0]["q"].float() - a[0]["k"].float().repeat_interleave(4, dim=1))
    assert 0.3 < float(d.std()) < 0.7


def test_extra_pages_add_table_columns_and_spare_blocks():
    wl = synth.Workload("s", batch=3, layers=1, hq=2, hkv=1, head_dim=64, ctx_lo=20, ctx_hi=40,
                        window=16, keep=4)
    base = synth.make_cache(wl, 5, "cpu", with_queries=False)
    more = synth.make_cache(wl, 5, "cpu", with_queries=False, extra_pages=4)
    assert more["max_blocks"] == base["max_blocks"] + 4
    assert more["num_blocks"] == base["num_blocks"] + 3 * 4
    assert int(more["free_top"][0]) == int(base["free_top"][0]) + 3 * 4
