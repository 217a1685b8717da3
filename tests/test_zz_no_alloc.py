"""kara_compact_noalloc: the compaction entry point that allocates no device memory.

Some callers cannot allocate device memory when they compress: a serving engine that gave all
free device memory to its KV block pool at start-up, or a C caller without a device allocator.
For them the library keeps the compaction plan in a fixed device array. This file is collected
last so that a run stopping at the first failure has already run every other test; it passes
alone in a fresh process as well as after the rest of the suite.
"""

import ctypes

import numpy as np
import pytest
import torch

from decode_kv_cache_kara_b200 import kara as K
from decode_kv_cache_kara_b200 import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu

WL = synth.WORKLOADS["layer"].with_(batch=5, ctx_lo=300, ctx_hi=900, window=200, keep=40,
                                    spare_blocks=64)


def run_both(cpu, keep, seq_ids=None):
    """The existing entry point and the allocation-free one on two copies of the same state."""
    a, b = H.to_device(cpu), H.to_device(cpu)
    sid = None if seq_ids is None else torch.tensor(seq_ids, dtype=torch.int32, device="cuda")
    keep_d = torch.from_numpy(keep).cuda()
    st_a = K.kara_compact(a["k"], a["v"], K.PagedPool.from_cache(a), WL.window, keep_d, seq_ids=sid)
    st_b = K.new_status()
    K.kara_compact_noalloc(b["k"], b["v"], K.PagedPool.from_cache(b), WL.window, keep_d,
                           seq_ids=sid, status=st_b)
    torch.cuda.synchronize()
    return a, b, K.read_status(st_a), K.read_status(st_b)


def assert_same_state(a, b):
    # compaction is bit-exact: the tolerance of the compaction tests is equality
    for key in ("block_table", "ctx_len", "free_top"):
        assert torch.equal(a[key], b[key]), key
    top = int(a["free_top"][0])
    assert torch.equal(a["free_list"][:top], b["free_list"][:top])
    bt = H.i32(a["block_table"])
    for layer in range(len(a["k"])):
        for pools in (("k", "k"), ("v", "v")):
            ga, gb = H.bits(a[pools[0]][layer]), H.bits(b[pools[1]][layer])
            for s in range(bt.shape[0]):
                n = int(a["ctx_len"][s])
                assert np.array_equal(H.logical_rows(ga, bt[s], n), H.logical_rows(gb, bt[s], n))


def test_noalloc_matches_kara_compact_on_two_calls_in_a_row():
    rng = np.random.default_rng(7)
    cpu = synth.make_cache(WL, 61, "cpu", layers=2)
    # first call: every sequence
    keep1 = np.stack([synth.random_keep(rng, WL.batch * WL.hkv, WL.window, WL.keep)
                      .reshape(WL.batch, WL.hkv, WL.keep) for _ in range(2)])
    a, b, sa, sb = run_both(cpu, keep1)
    assert sa == 0 and sb == 0
    assert_same_state(a, b)
    # second call, right after, on a different subset and keep (the array holds the first
    # call's plan; nothing of it may leak into the second)
    keep2 = np.stack([synth.random_keep(rng, 2 * WL.hkv, WL.window, WL.keep)
                      .reshape(2, WL.hkv, WL.keep) for _ in range(2)])
    a2, b2, sa, sb = run_both(cpu, keep2, seq_ids=[1, 4])
    assert sa == 0 and sb == 0
    assert_same_state(a2, b2)


def test_noalloc_rejects_plans_larger_than_its_array():
    cpu = synth.make_cache(WL, 62, "cpu", layers=1)
    dev = H.to_device(cpu)
    pool = K.PagedPool.from_cache(dev)
    limit = K.lib().kara_compact_noalloc
    null = ctypes.c_void_p(0)
    arr = K._layers(dev["k"], dev["v"])
    ps = pool.c_struct()
    # 4 * (144 + 12 R + R * ceil((15 + k) / 16)) > 64 KiB for R = 4096, k = 204
    rc = limit(arr, 1, ctypes.byref(ps), null, 4096, 1024, 204, null, null, null)
    assert rc == K.ERR_WORKSPACE
