"""Parity on the step and 8B-GQA workloads' shapes, the whole path on the GPU.

Every per-sequence size is the workload's own; only the batch and the layer count are cut so
that the oracle can check the results:
- step: 28 q / 4 kv heads, d=128, ragged contexts 2K-16K, W=1024 (fused scorer on clusters of
  8), keep 204, Token2Chunk anchors 50 % / gap 8 / widen 1; 5 sequences, 3 layers;
- gqa8b: 32 q / 8 kv heads, d=128, ragged contexts 8K-32K, W=2048 (fused scorer on clusters of
  16), keep 409; 3 sequences, 2 layers.
Each layer is scored, selected and expanded, all layers are compacted in one call, and layer
0 of the compacted cache is decoded. Checks: sampled score rows against the oracle, select and
Token2Chunk exactly on those rows, compaction bit-exact on every layer and sequence, decode on
every sequence.
"""
import math

import numpy as np
import pytest
import torch

from decode_kv_cache_kara_b200 import kara as K
from decode_kv_cache_kara_b200 import synth
from oracle import decode as od
from oracle import kara as ok
from tests import helpers as H

pytestmark = pytest.mark.gpu

CASES = {
    "step": (synth.WORKLOADS["step"].with_(batch=5, layers=3), 1234 + 2),
    "gqa8b": (synth.WORKLOADS["gqa8b"].with_(batch=3, layers=2), 1234 + 3),
}


def _pool_f64(b):
    return torch.from_numpy(b).view(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_config_path_sampled(name):
    wl, seed = CASES[name]
    cache = synth.make_cache(wl, seed, "cuda")
    kb = [H.bits(t) for t in cache["k"]]
    vb = [H.bits(t) for t in cache["v"]]
    bt0, cl0 = H.i32(cache["block_table"]), H.i32(cache["ctx_len"])
    fl0, top0 = H.i32(cache["free_list"]), int(cache["free_top"][0])
    qw = [q.cpu() for q in cache["q_win"]]
    pool = K.PagedPool.from_cache(cache)
    na = wl.anchor_frac
    status = K.new_status()
    keep = torch.empty((wl.layers, wl.batch, wl.hkv, wl.keep), dtype=torch.int32, device="cuda")
    scores, sels = [], []
    for layer in range(wl.layers):
        n0 = K.kara_launch_count()
        sc = K.kara_score(cache["q_win"][layer], cache["k"][layer], pool, wl.window, status=status)
        # the fused kernel (and the split-item sum when a cluster's range ends inside an item);
        # the two-pass path takes three launches
        assert K.kara_launch_count() - n0 <= 2
        sel = K.kara_select(sc, wl.keep)
        K.kara_token2chunk(sc, sel, na, wl.gap_limit, wl.widen, keep=keep[layer])
        scores.append(sc)
        sels.append(sel)
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    scale = 1 / math.sqrt(wl.head_dim)

    # scores, select and Token2Chunk on sampled rows of every layer
    rng = np.random.default_rng(3)
    for layer in range(wl.layers):
        s = H.f64(scores[layer])
        assert np.allclose(s.sum(-1), wl.window * wl.group, rtol=1e-4)
        kf = _pool_f64(kb[layer])
        sl, kp = H.i32(sels[layer]), H.i32(keep[layer])
        for r, g in zip(rng.integers(0, wl.batch, 2), rng.integers(0, wl.hkv, 2)):
            n = int(cl0[r])
            slots = ok.window_slots(n, wl.window)
            kw = ok.gather_rows(kf, bt0[r], slots, wl.page)[:, g:g + 1]
            heads = list(range(g * wl.group, (g + 1) * wl.group))
            q = qw[layer][r][:, heads].double().numpy()
            H.assert_scores_close(s[r, g], ok.window_scores(q, kw, scale)[0])
            assert np.array_equal(sl[r, g], ok.select_topk(s[r, g], wl.keep))
            assert np.array_equal(kp[r, g], ok.token2chunk(s[r, g], sl[r, g],
                                                           ok.anchors_for(na, wl.keep),
                                                           wl.gap_limit, wl.widen))

    # compaction of all layers, bit-exact
    ws = torch.empty(K.kara_workspace_bytes(K.OP_COMPACT, pool, wl.batch, wl.window, 0, wl.keep),
                     dtype=torch.uint8, device="cuda")
    K.kara_compact(cache["k"], cache["v"], pool, wl.window, keep, workspace=ws, status=status)
    torch.cuda.synchronize()
    assert K.read_status(status) == 0
    st, kpo, vpo, bt, cl, fl, top, _ = ok.compact(kb, vb, bt0, cl0, fl0, top0,
                                                  list(range(wl.batch)), wl.window, H.i32(keep),
                                                  wl.page)
    assert st == ok.OK
    assert np.array_equal(H.i32(cache["block_table"]), bt)
    assert np.array_equal(H.i32(cache["ctx_len"]), cl)
    assert int(cache["free_top"][0]) == top
    assert np.array_equal(H.i32(cache["free_list"])[:top], fl[:top])
    for layer in range(wl.layers):
        kg, vg = H.bits(cache["k"][layer]), H.bits(cache["v"][layer])
        for b in range(wl.batch):
            n = int(cl[b])
            assert np.array_equal(H.logical_rows(kg, bt[b], n), H.logical_rows(kpo[layer], bt[b], n))
            assert np.array_equal(H.logical_rows(vg, bt[b], n), H.logical_rows(vpo[layer], bt[b], n))

    # decode of layer 0 over the compacted cache, every sequence
    out = K.paged_decode_attn(cache["q_dec"], cache["k"][0], cache["v"][0], pool)
    torch.cuda.synchronize()
    ref = od.decode_attention(H.f64(cache["q_dec"]), H.f64(cache["k"][0]), H.f64(cache["v"][0]),
                              bt, cl, scale, wl.page)
    assert np.allclose(H.f64(out), ref, atol=2e-2, rtol=1e-2)


def test_gqa8b_free_and_reuse():
    # The 8B-GQA workload's shapes (32 q / 8 kv heads, ragged 8K-32K contexts, W=2048, keep
    # 409; 3 sequences, 1 layer): a compaction, then W new tokens per sequence whose pages come
    # from the free list top (so they reuse blocks the first compaction freed), then a second
    # compaction over the new window. Both bit-exact against the oracle.
    wl = synth.WORKLOADS["gqa8b"].with_(batch=3, layers=1)
    cpu = synth.make_cache(wl, 1234 + 3, "cpu", with_queries=False,
                           extra_pages=wl.window // 16 + 2)
    dev = H.to_device(cpu)
    pool = K.PagedPool.from_cache(dev)
    rng = np.random.default_rng(21)
    ids = list(range(wl.batch))

    def compact_both(state, keep):
        ref = ok.compact([H.bits(state["k"][0])], [H.bits(state["v"][0])],
                         H.i32(state["block_table"]), H.i32(state["ctx_len"]),
                         H.i32(state["free_list"]), int(state["free_top"][0]), ids, wl.window,
                         keep, wl.page)
        st = K.kara_compact(dev["k"], dev["v"], pool, wl.window, torch.from_numpy(keep).cuda())
        torch.cuda.synchronize()
        assert K.read_status(st) == 0 and ref[0] == ok.OK
        _, kp, vp, bt, cl, fl, top, fresh = ref
        assert np.array_equal(H.i32(dev["block_table"]), bt)
        assert np.array_equal(H.i32(dev["ctx_len"]), cl)
        assert int(dev["free_top"][0]) == top
        assert np.array_equal(H.i32(dev["free_list"])[:top], fl[:top])
        kg, vg = H.bits(dev["k"][0]), H.bits(dev["v"][0])
        for b in ids:
            n = int(cl[b])
            assert np.array_equal(H.logical_rows(kg, bt[b], n), H.logical_rows(kp[0], bt[b], n))
            assert np.array_equal(H.logical_rows(vg, bt[b], n), H.logical_rows(vp[0], bt[b], n))
        return kp, vp, bt, cl, fl, top, fresh

    keep1 = synth.random_keep(rng, wl.batch * wl.hkv, wl.window, wl.keep).reshape(
        1, wl.batch, wl.hkv, wl.keep)
    kp, vp, bt, cl, fl, top, _ = compact_both(cpu, keep1)
    old = H.i32(cpu["block_table"])
    freed = set(old[old >= 0].tolist()) - set(bt[bt >= 0].tolist())
    assert len(freed) >= wl.batch * (wl.window // 16)

    # W new tokens per sequence: pages popped from the free list top (sequence order), their
    # K/V rows drawn from N(0, 1); the same on the host state and on the device
    bt, cl, fl = bt.copy(), cl.copy(), fl.copy()
    kp0, vp0 = kp[0].copy(), vp[0].copy()
    popped = []
    for b in ids:
        n = int(cl[b])
        for p in range((n + 15) // 16, (n + wl.window + 15) // 16):
            top -= 1
            bt[b, p] = fl[top]
            popped.append(int(fl[top]))
        slots = np.arange(n, n + wl.window)
        rows = rng.standard_normal((2, wl.window, wl.hkv, wl.head_dim)).astype(np.float32)
        kb = torch.from_numpy(rows[0]).to(torch.bfloat16).view(torch.int16).numpy()
        vb = torch.from_numpy(rows[1]).to(torch.bfloat16).view(torch.int16).numpy()
        kp0[bt[b][slots // 16], slots % 16] = kb
        vp0[bt[b][slots // 16], slots % 16] = vb
        cl[b] = n + wl.window
    assert set(popped) & freed                      # the new pages reuse freed blocks
    state2 = {"k": [torch.from_numpy(kp0).view(torch.bfloat16)],
              "v": [torch.from_numpy(vp0).view(torch.bfloat16)],
              "block_table": torch.from_numpy(bt.astype(np.int32)),
              "ctx_len": torch.from_numpy(cl.astype(np.int32)),
              "free_list": torch.from_numpy(fl.astype(np.int32)),
              "free_top": torch.tensor([top], dtype=torch.int32)}
    for key in ("block_table", "ctx_len", "free_list", "free_top"):
        dev[key].copy_(state2[key].cuda())
    dev["k"][0].copy_(state2["k"][0].cuda())
    dev["v"][0].copy_(state2["v"][0].cuda())
    keep2 = synth.random_keep(rng, wl.batch * wl.hkv, wl.window, wl.keep).reshape(
        1, wl.batch, wl.hkv, wl.keep)
    _, _, bt2, _, _, _, fresh2 = compact_both(state2, keep2)
    reused = set(x for ids_ in fresh2.values() for x in ids_) & freed
    assert reused                                    # the second compaction pops freed blocks too
