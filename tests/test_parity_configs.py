"""Parity on the step and 8B-GQA workloads' shapes, the whole path on the GPU.

Every per-sequence size is the workload's own; only the batch and the layer count are cut so
that the oracle can check the results:
- step: 28 q / 4 kv heads, d=128, ragged contexts 2K-16K, W=1024 (fused cluster scorer),
  keep 204, Token2Chunk anchors 50 % / gap 8 / widen 1; 5 sequences, 3 layers;
- gqa8b: 32 q / 8 kv heads, d=128, ragged contexts 8K-32K, W=2048 (two-pass scorer),
  keep 409; 3 sequences, 2 layers.
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
        sc = K.kara_score(cache["q_win"][layer], cache["k"][layer], pool, wl.window, status=status)
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
