"""The multi-GPU path's host logic on CPU: world size 2 over gloo.

Sequences are independent, so every rank compresses its own batch (weak scaling) with no
collective on the data path; only the step time is reduced (max over ranks) and the whole-job
value counts every rank's window tokens. The ranks here run the oracle step on their shards.
"""

import math
import os
import time

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from decode_kv_cache_kara_b200 import synth
from oracle import kara as ok

WL = synth.WORKLOADS["tiny"].with_(batch=2)


def _rank_main(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cache = synth.make_cache(WL, bench.rank_seed(rank), "cpu")
        t0 = time.perf_counter()
        q = cache["q_win"][0].double().numpy()
        kp = cache["k"][0].double().numpy()
        bt = cache["block_table"].numpy().astype(np.int64)
        cl = cache["ctx_len"].numpy().astype(np.int64)
        s = ok.score_batch(q, kp, bt, cl, list(range(WL.batch)), WL.window,
                           1 / math.sqrt(WL.head_dim), WL.page)
        sel = ok.select_batch(s, WL.keep)
        keep = ok.token2chunk_batch(s, sel, ok.anchors_for(WL.anchor_frac, WL.keep),
                                    WL.gap_limit, WL.widen)
        st, *_ = ok.compact([cache["k"][0].view(torch.int16).numpy()],
                            [cache["v"][0].view(torch.int16).numpy()], bt, cl,
                            cache["free_list"].numpy(), int(cache["free_top"][0]),
                            list(range(WL.batch)), WL.window, keep[None], WL.page)
        local_ms = (time.perf_counter() - t0) * 1e3 + 5.0 * rank     # ranks differ in time
        worst = bench.max_over_ranks(local_ms, "cpu", world)
        shards = [None] * world
        dist.all_gather_object(shards, float(cache["k"][0].float().sum()))
        value = bench.whole_job_value(WL.batch * WL.window, world, worst)
        np.save(os.path.join(outdir, f"r{rank}.npy"),
                np.array([st, local_ms, worst, value, shards[0], shards[1]]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_ranks_shard_sequences_and_reduce_the_step_time(tmp_path):
    port = 29500 + os.getpid() % 1000
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    r0 = np.load(tmp_path / "r0.npy")
    r1 = np.load(tmp_path / "r1.npy")
    assert r0[0] == 0 and r1[0] == 0                       # both shards compacted
    assert r0[2] == r1[2] == max(r0[1], r1[1])             # same max-over-ranks time
    assert r0[3] == pytest.approx(2 * WL.batch * WL.window / (r0[2] / 1e3))
    assert r0[4] != r0[5]                                  # the ranks hold different batches
    assert bench.rank_seed(0) == 1236 and bench.rank_seed(1) != bench.rank_seed(0)
