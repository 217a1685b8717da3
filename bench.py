"""Throughput benchmark of the Kara decode-time compression step on B200.

One step = one pass of the whole hot path over one batch of the "layer" workload (one
7B-class layer, batch 32, 28 query / 4 KV heads, d = 128, 4096-token paged caches, window
1024, keep 204): kara_score -> kara_select_chunks (select and Token2Chunk in one kernel) ->
kara_compact -> paged_decode_attn over the compressed cache, then the block table, lengths and free list are
restored so that every step sees the same input. Metric: compressed KV tokens per second
(window tokens of all due sequences / step time), whole job over all ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU (torchrun, one rank per GPU): sequences are independent, so every rank compresses
its own batch (weak scaling) with no collective on the data path; the step time is the max
over ranks. ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from decode_kv_cache_kara_b200 import synth  # noqa: E402

METRIC = "compressed KV tokens/sec on 1 B200; % tensor/HBM roofline per kernel"
UNIT = "tokens/s"
WORKLOAD = synth.WORKLOADS["layer"]
WORKLOAD_DESC = ("layer: one 7B-class layer, batch 32, 28 query / 4 KV heads, head_dim 128, "
                 "4096-token paged caches (page 16), window W=1024 (last 1024 tokens), keep 204 "
                 "(20%), Token2Chunk anchors 50% / gap 8 / widen 1, then paged GQA decode over "
                 "the compressed cache")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def captured_traffic(op: str):
    """DRAM bytes per launch of `op` from the committed ncu summary (profiles/traffic.txt),
    or None when the kernel source changed since the capture (its sha256 no longer matches)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        parts = line.split()
        if len(parts) != 4 or line.startswith("#") or parts[0] != op:
            continue
        src = os.path.join(ROOT, "decode_kv_cache_kara_b200", parts[1])
        if not os.path.exists(src):
            return None
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return int(parts[3]) if digest == parts[2] else None
    return None


def rank_seed(rank: int) -> int:
    """Seed of a rank's batch: the layer workload's seed (1234 + config index 1), offset per
    rank so that every rank compresses its own, independent sequences."""
    return 1234 + 1 + 1000 * rank


def max_over_ranks(x: float, device, world: int) -> float:
    """The maximum of a per-rank scalar over all ranks (the step time of the whole job)."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(tokens_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: window tokens of every rank per second of the slowest rank."""
    return tokens_per_rank_step * world / (ms_per_step / 1e3)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        load = [s for s in sm if smax and s > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------
class Step:
    """One compression step of the whole path on a device-resident workload."""

    def __init__(self, cache: dict, wl: synth.Workload):
        from decode_kv_cache_kara_b200 import kara as K
        self.K = K
        self.wl = wl
        self.c = cache
        dev = cache["k"][0].device
        # the pool bookkeeping as views into one int32 buffer, so that the per-step restore
        # is a single copy
        names = ("block_table", "ctx_len", "free_list", "free_top")
        sizes = [cache[n].numel() for n in names]
        self.book = torch.empty(sum(sizes), dtype=torch.int32, device=dev)
        off = 0
        for n, sz in zip(names, sizes):
            view = self.book[off:off + sz].view(cache[n].shape)
            view.copy_(cache[n])
            cache[n] = view
            off += sz
        self.saved_book = self.book.clone()
        self.pool = K.PagedPool.from_cache(cache)
        self.status = K.new_status(dev)
        r, hq = wl.batch, wl.hq
        self.scores = torch.empty((r, wl.hkv, wl.window), dtype=torch.float32, device=dev)
        self.sel = torch.empty((r, wl.hkv, wl.keep), dtype=torch.int32, device=dev)
        self.keep = torch.empty((1, r, wl.hkv, wl.keep), dtype=torch.int32, device=dev)
        self.out = torch.empty((wl.batch, hq, wl.head_dim), dtype=torch.bfloat16, device=dev)
        ws = max(K.kara_workspace_bytes(K.OP_SCORE, self.pool, r, wl.window, hq),
                 K.kara_workspace_bytes(K.OP_COMPACT, self.pool, r, wl.window, 0, wl.keep),
                 K.kara_workspace_bytes(K.OP_DECODE, self.pool, 0, 0, hq, 0))
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.na = wl.anchor_frac
        # scoring: the fused cluster kernel for windows of 128/256/512/1024 keys (plus the
        # split-item sum when a cluster range ends inside an item), else two passes and a
        # merge; select + Token2Chunk in one kernel; compaction plan + gather; decode + combine
        self.score_fused = wl.window in (128, 256, 512, 1024)

    def restore(self):
        self.book.copy_(self.saved_book, non_blocking=True)

    def run(self, events=None, restore=True):
        K, wl, c = self.K, self.wl, self.c
        rec = (lambda i: events[i].record()) if events is not None else (lambda i: None)
        rec(0)
        K.kara_score(c["q_win"][0], c["k"][0], self.pool, wl.window, scores=self.scores,
                     workspace=self.ws, status=self.status)
        rec(1)
        K.kara_select_chunks(self.scores, wl.keep, self.na, wl.gap_limit, wl.widen,
                             keep=self.keep[0], sel=self.sel)
        rec(2)
        K.kara_compact(c["k"], c["v"], self.pool, wl.window, self.keep, workspace=self.ws,
                       status=self.status)
        rec(3)
        K.paged_decode_attn(c["q_dec"], c["k"][0], c["v"][0], self.pool, out=self.out,
                            workspace=self.ws, status=self.status)
        rec(4)
        if restore:
            self.restore()


def algorithmic_work(wl: synth.Workload, cache: dict) -> dict:
    """Per-launch algorithmic flops / bytes of each op (inputs before the step)."""
    ctx = cache["ctx_len"].cpu().numpy().astype(np.int64)
    r, W, d, hq, hkv, k = wl.batch, wl.window, wl.head_dim, wl.hq, wl.hkv, wl.keep
    score_flops = 2.0 * W * W * d * hq * r                       # one Q K^T, useful
    off = (ctx - W) % wl.page
    rows = (hkv * (k + off)).sum()                               # head-rows copied
    compact_bytes = float(rows * d * 2 * 2 * 2)                  # K and V, read + write
    n_after = ctx - W + k
    decode_bytes = float(n_after.sum() * hkv * d * 2 * 2 + 2 * r * hq * d * 2)
    return {"score_flops": score_flops, "compact_bytes": compact_bytes,
            "decode_bytes": decode_bytes}


def time_cpu_oracle_sample(cache_cpu: dict, wl: synth.Workload, units: int = 1, seed: int = 0):
    """The oracle as it stands on one (sequence, KV head) unit per call: score (its G query
    heads), select, Token2Chunk, compaction of its rows, decode of its G query heads.
    Returns (seconds, window tokens equivalent)."""
    from oracle import decode as od
    from oracle import kara as ok
    rng = np.random.default_rng(seed)
    bt = cache_cpu["block_table"].numpy().astype(np.int64)
    cl = cache_cpu["ctx_len"].numpy().astype(np.int64)
    scale = 1 / math.sqrt(wl.head_dim)
    t0 = time.perf_counter()
    for _ in range(units):
        b = int(rng.integers(0, wl.batch))
        g = int(rng.integers(0, wl.hkv))
        heads = list(range(g * wl.group, (g + 1) * wl.group))
        n = int(cl[b])
        slots = ok.window_slots(n, wl.window)
        blocks = bt[b][slots // wl.page]
        kw = cache_cpu["k"][0][blocks, slots % wl.page][:, g:g + 1].double().numpy()
        qw = cache_cpu["q_win"][0][b][:, heads].double().numpy()
        s = ok.window_scores(qw, kw, scale)[0]
        sel = ok.select_topk(s, wl.keep)
        keep = ok.token2chunk(s, sel, ok.anchors_for(wl.anchor_frac, wl.keep), wl.gap_limit,
                              wl.widen)
        # compaction of this head's rows (one layer, one sequence, one KV head)
        kb = cache_cpu["k"][0].view(torch.int16).numpy()
        vb = cache_cpu["v"][0].view(torch.int16).numpy()
        sub_k = kb[:, :, g:g + 1].copy()
        sub_v = vb[:, :, g:g + 1].copy()
        st, kp, vp, bt2, cl2, _, _, _ = ok.compact(
            [sub_k], [sub_v], bt, cl, cache_cpu["free_list"].numpy(),
            int(cache_cpu["free_top"][0]), [b], wl.window, keep[None, None, None, :], wl.page)
        kd = torch.from_numpy(kp[0]).view(torch.bfloat16)
        vd = torch.from_numpy(vp[0]).view(torch.bfloat16)
        nn = int(cl2[b])
        sl = np.arange(nn)
        kk = kd[bt2[b][sl // wl.page], sl % wl.page].double().numpy()     # [nn, 1, d]
        vv = vd[bt2[b][sl // wl.page], sl % wl.page].double().numpy()
        q = cache_cpu["q_dec"][b:b + 1, heads].double().numpy()           # [1, G, d]
        # the compacted sequence as one block of nn slots
        od.decode_attention(q, kk[None], vv[None], np.array([[0]]), np.array([nn]), scale, nn)
    dt = time.perf_counter() - t0
    return dt, units * wl.window / wl.hkv


def e2e_run(cache: dict, wl: synth.Workload, steps: int, warmup: int) -> dict:
    """The same step through the public API with HOST inputs: every step copies the inputs from
    pinned host memory to the device and reads the results back."""
    from decode_kv_cache_kara_b200 import kara as K
    dev = cache["k"][0].device
    names_in = ["q_win", "k", "v", "q_dec", "block_table", "ctx_len", "free_list", "free_top"]
    host = {}
    for n in names_in:
        val = cache[n]
        host[n] = ([t.cpu().pin_memory() for t in val] if isinstance(val, list)
                   else val.cpu().pin_memory())
    dcache = {n: ([torch.empty_like(t, device=dev) for t in host[n]] if isinstance(host[n], list)
                  else torch.empty_like(host[n], device=dev)) for n in names_in}
    dcache["num_blocks"] = cache["num_blocks"]
    out_host = {"out": torch.empty((wl.batch, wl.hq, wl.head_dim), dtype=torch.bfloat16).pin_memory(),
                "keep": torch.empty((1, wl.batch, wl.hkv, wl.keep), dtype=torch.int32).pin_memory(),
                "block_table": torch.empty_like(host["block_table"]).pin_memory(),
                "ctx_len": torch.empty_like(host["ctx_len"]).pin_memory()}

    def h2d():
        for n in names_in:
            if isinstance(host[n], list):
                for d_, h_ in zip(dcache[n], host[n]):
                    d_.copy_(h_, non_blocking=True)
            else:
                dcache[n].copy_(host[n], non_blocking=True)

    h2d_bytes = sum(t.numel() * t.element_size() for n in names_in
                    for t in (host[n] if isinstance(host[n], list) else [host[n]]))
    d2h_bytes = sum(t.numel() * t.element_size() for t in out_host.values())
    h2d()
    step = Step(dcache, wl)

    def one():
        h2d()                       # the next step's copy replaces the compacted state
        step.run(restore=False)
        out_host["out"].copy_(step.out, non_blocking=True)
        out_host["keep"].copy_(step.keep, non_blocking=True)
        out_host["block_table"].copy_(dcache["block_table"], non_blocking=True)
        out_host["ctx_len"].copy_(dcache["ctx_len"], non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return {"ms_per_step": ms, "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes}


def lacache_run(dev, batch: int, reps: int = 5, warmup: int = 3) -> dict:
    """One LaCache ladder-compaction pass (all 32 layers, 64K -> 8192 slots per layer) on the
    LaCache workload, timed with CUDA events; the block table, lengths and free list are
    restored between passes (the pass only writes fresh blocks), so every pass sees the same
    full cache."""
    from decode_kv_cache_kara_b200 import kara as K
    wl = synth.WORKLOADS["lacache"].with_(batch=batch)
    ex = wl.extra
    cache = synth.make_cache(wl, 1234 + 4, dev, with_queries=False)
    pool = K.PagedPool.from_cache(cache)
    saved = {k: cache[k].clone() for k in ("block_table", "ctx_len", "free_list", "free_top")}
    ws = torch.empty(K.kara_workspace_bytes(K.OP_LACACHE, pool, wl.batch, 0, 0, ex["budget"]),
                     dtype=torch.uint8, device=dev)
    status = K.new_status(dev)

    def one():
        K.lacache_compact(cache["k"], cache["v"], pool, ex["span"], ex["overlap"], ex["rung"],
                          ex["budget"], ex["sink"], ex["recent"], workspace=ws, status=status)

    def restore():
        for k, t in saved.items():
            cache[k].copy_(t)

    for _ in range(warmup):
        one()
        restore()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        one()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
        restore()
    torch.cuda.synchronize()
    st = K.read_status(status)
    ms = sum(times) / len(times)
    # every layer keeps `budget` slots: K and V rows of [Hkv, d] read once and written once
    nbytes = 2 * 2 * wl.batch * wl.layers * ex["budget"] * wl.hkv * wl.head_dim * 2
    del cache, saved, ws
    torch.cuda.empty_cache()
    return {"ms": ms, "bound": "hbm", "gbs": nbytes / ms / 1e6, "bytes": nbytes, "status": st,
            "workload": f"lacache: batch {wl.batch}, 32 layers, 8 KV heads, d=128, 64K-token "
                        f"caches, S=8, O=4, rung 64, budget 8192 per layer; one pass (all layers)"}


def variants_run(step, reps: int = 10) -> dict:
    """The score and selection variants on the layer workload (its window queries and cache,
    not changed by them): kara_score_ex with the mean and with the max aggregation, and the
    selection shared across KV heads (head sums, select, Token2Chunk, expansion to every
    head). Average times with CUDA events over `reps` calls after one untimed call."""
    K, wl, c = step.K, step.wl, step.c
    tot = torch.empty((wl.batch, wl.window), dtype=torch.float32, device=step.scores.device)
    shared = torch.empty((wl.batch, wl.keep), dtype=torch.int32, device=tot.device)
    sel = torch.empty((wl.batch, wl.keep), dtype=torch.int32, device=tot.device)

    def score(agg):
        K.kara_score_ex(c["q_win"][0], c["k"][0], step.pool, wl.window, agg=agg,
                        scores=step.scores, workspace=step.ws, status=step.status)

    def shared_select():
        K.kara_sum_heads(step.scores, out=tot)
        K.kara_select(tot, wl.keep, sel=sel)
        K.kara_token2chunk(tot, sel, step.na, wl.gap_limit, wl.widen, keep=shared)
        K.kara_expand_keep(shared, wl.hkv, keep=step.keep[0])

    out = {}
    def select_then_chunks():
        K.kara_select(step.scores, wl.keep, sel=step.sel)
        K.kara_token2chunk(step.scores, step.sel, step.na, wl.gap_limit, wl.widen,
                           keep=step.keep[0])

    for name, fn in (("score_mean_ms", lambda: score(K.AGG_MEAN)),
                     ("score_max_ms", lambda: score(K.AGG_MAX)),
                     ("shared_select_ms", shared_select),
                     ("select_then_token2chunk_ms", select_then_chunks)):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        out[name] = e0.elapsed_time(e1) / reps
    # selection, Token2Chunk and compaction: two calls (three kernels) against kara_compress
    # (plan + one fused kernel); the bookkeeping is restored between repetitions, untimed
    def compact_pair():
        K.kara_select_chunks(step.scores, wl.keep, step.na, wl.gap_limit, wl.widen,
                             keep=step.keep[0])
        K.kara_compact(c["k"], c["v"], step.pool, wl.window, step.keep, workspace=step.ws,
                       status=step.status)

    def compress():
        K.kara_compress(step.scores[None], c["k"], c["v"], step.pool, wl.window, wl.keep, step.na,
                        wl.gap_limit, wl.widen, keep=step.keep, workspace=step.ws,
                        status=step.status)

    for name, fn in (("select_chunks_then_compact_ms", compact_pair), ("compress_ms", compress)):
        fn()
        step.restore()
        torch.cuda.synchronize()
        total = 0.0
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            step.restore()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        out[name] = total / reps
    out["status"] = K.read_status(step.status)
    out["note"] = ("layer workload; max runs the two-pass kernels (a max, not a sum, per key); "
                   "shared = head sums, one select + Token2Chunk per (sequence, layer), keep "
                   "copied to the 4 KV heads; select_then_token2chunk = the two calls the "
                   "step's fused kara_select_chunks replaces")
    return out


def decode_loop_run(dev, steps: int = 300, period: int = 100, warm: int = 20) -> dict:
    """The decode loop on the layer workload's shapes (batch 32, 28 query / 4 KV heads, d=128,
    4096-token contexts, W=1024, keep 204, one layer): every step kara_step_begin,
    kara_decode_append and kara_step_end; every `period` steps the due sequences (tail >= W)
    are compressed (kara_score_ring, kara_select_chunks, kara_compact,
    kara_reset_tails). Tails start spread over [0, W) and the query ring holds seeded queries,
    as in the middle of a generation. Timed with CUDA events per step; a check step includes
    the host read of the due count that sizes its compression."""
    from decode_kv_cache_kara_b200 import kara as K
    wl = WORKLOAD
    W, B = wl.window, wl.batch
    cache = synth.make_cache(wl, 1234 + 5, dev, with_queries=False,
                             extra_pages=(steps + warm) // wl.page + 2)
    pool = K.PagedPool.from_cache(cache)
    k0, v0 = cache["k"][0], cache["v"][0]
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + 6)
    ring = torch.randn((B, 2 * W, wl.hq, wl.head_dim), generator=gen, device=dev).to(torch.bfloat16)
    tail = torch.randint(0, W, (B,), generator=gen, device=dev, dtype=torch.int32)
    inputs = [[torch.randn(shape, generator=gen, device=dev).to(torch.bfloat16)
               for shape in ((B, wl.hq, wl.head_dim), (B, wl.hkv, wl.head_dim),
                             (B, wl.hkv, wl.head_dim))] for _ in range(16)]
    out = torch.empty((B, wl.hq, wl.head_dim), dtype=torch.bfloat16, device=dev)
    ws_dec = torch.empty(K.kara_workspace_bytes(K.OP_DECODE, pool, 0, 0, wl.hq, 0),
                         dtype=torch.uint8, device=dev)
    ws_sc = torch.empty(K.kara_workspace_bytes(K.OP_SCORE, pool, B, W, wl.hq), dtype=torch.uint8,
                        device=dev)
    ws_cp = torch.empty(K.kara_workspace_bytes(K.OP_COMPACT, pool, B, W, 0, wl.keep),
                        dtype=torch.uint8, device=dev)
    scores = torch.empty((B, wl.hkv, W), dtype=torch.float32, device=dev)
    sel = torch.empty((B, wl.hkv, wl.keep), dtype=torch.int32, device=dev)
    keep = torch.empty((1, B, wl.hkv, wl.keep), dtype=torch.int32, device=dev)
    due = torch.zeros(B, dtype=torch.int32, device=dev)
    due_count = torch.zeros(1, dtype=torch.int32, device=dev)
    status = K.new_status(dev)
    na = wl.anchor_frac

    def step(t, check):
        q, kn, vn = inputs[t % len(inputs)]
        K.kara_step_begin(pool, status)
        K.kara_decode_append(q, kn, vn, k0, v0, pool, ring, W, out=out, workspace=ws_dec,
                             status=status)
        K.kara_step_end(pool, tail, W, check, due, due_count)
        if not check:
            return 0
        cnt = int(due_count.item())
        if cnt:
            seq = due[:cnt]
            K.kara_score_ring(ring, k0, pool, W, seq, cnt, scores=scores[:cnt], workspace=ws_sc,
                              status=status)
            K.kara_select_chunks(scores[:cnt], wl.keep, na, wl.gap_limit, wl.widen,
                                 keep=keep[0, :cnt])
            K.kara_compact([k0], [v0], pool, W, keep[:, :cnt], seq_ids=seq, workspace=ws_cp,
                           status=status)
            K.kara_reset_tails(tail, seq, cnt)
        return cnt

    for t in range(warm):
        step(t, False)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    dues, checks = [], []
    for t in range(steps):
        check = (t + 1) % period == 0
        ev[t][0].record()
        n = step(warm + t, check)
        ev[t][1].record()
        if check:
            dues.append(n)
            checks.append(t)
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev]
    plain = sorted(m for t, m in enumerate(ms) if t not in checks)
    st = K.read_status(status)
    total = sum(ms)
    return {"steps": steps, "period": period, "ms_per_step": total / steps,
            "decode_step_ms": plain[len(plain) // 2],
            "check_step_ms": [ms[t] for t in checks], "due_per_check": dues,
            "tokens_per_s": B * steps / (total / 1e3), "status": st,
            "workload": f"decode loop: batch {B}, 28 query / 4 KV heads, d=128, 4096-token "
                        f"contexts, W={W}, keep {wl.keep}, one layer, check every {period} "
                        f"steps, tails spread over [0, W)"}


def lacache_loop_run(dev, steps: int = 200, period: int = 100, warm: int = 10) -> dict:
    """LaCache inside the decode loop on the layer workload's shapes with 4 layers (batch 32,
    28 query / 4 KV heads, d=128, 4096-token contexts): every step kara_step_begin, one
    kara_decode_append per layer and kara_step_end with the capacity trigger; the ladder
    (S = 2, O = 1, rung 64, sink 64, recent 64, budget 2048 per layer, so capacity
    64 + 64 + 1920 * 4 / 2 = 3968 slots) runs on the sequences due at a check step. Timed with
    CUDA events per step; a check step includes the host read of the due count."""
    from decode_kv_cache_kara_b200 import kara as K
    wl = WORKLOAD.with_(layers=4)
    B, L = wl.batch, wl.layers
    span, overlap, rung, budget, sink, recent = 2, 1, 64, 2048, 64, 64
    cap = sink + recent + (budget - sink - recent) * L // span
    # spare blocks: the steps' new pages, and a ladder pass pops budget / 16 fresh blocks per
    # due sequence before it frees the old ones
    cache = synth.make_cache(wl, 1234 + 7, dev, with_queries=False,
                             extra_pages=(steps + warm) // wl.page + 2 + budget // wl.page)
    pool = K.PagedPool.from_cache(cache)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + 8)
    inputs = [[torch.randn(shape, generator=gen, device=dev).to(torch.bfloat16)
               for shape in ((B, wl.hq, wl.head_dim), (B, wl.hkv, wl.head_dim),
                             (B, wl.hkv, wl.head_dim))] for _ in range(8)]
    out = torch.empty((B, wl.hq, wl.head_dim), dtype=torch.bfloat16, device=dev)
    ws_dec = torch.empty(K.kara_workspace_bytes(K.OP_DECODE, pool, 0, 0, wl.hq, 0),
                         dtype=torch.uint8, device=dev)
    ws_lac = torch.empty(K.kara_workspace_bytes(K.OP_LACACHE, pool, B, 0, 0, budget),
                         dtype=torch.uint8, device=dev)
    due = torch.zeros(B, dtype=torch.int32, device=dev)
    due_count = torch.zeros(1, dtype=torch.int32, device=dev)
    status = K.new_status(dev)

    def step(t, check):
        q, kn, vn = inputs[t % len(inputs)]
        K.kara_step_begin(pool, status)
        for layer in range(L):
            K.kara_decode_append(q, kn, vn, cache["k"][layer], cache["v"][layer], pool, out=out,
                                 workspace=ws_dec, status=status)
        K.kara_step_end(pool, None, 0, check, due, due_count, capacity=cap)
        if not check:
            return 0
        cnt = int(due_count.item())
        if cnt:
            K.lacache_compact(cache["k"], cache["v"], pool, span, overlap, rung, budget, sink,
                              recent, seq_ids=due[:cnt], workspace=ws_lac, status=status)
        return cnt

    for t in range(warm):
        step(t, False)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    dues, checks = [], []
    for t in range(steps):
        check = (t + 1) % period == 0
        ev[t][0].record()
        n = step(warm + t, check)
        ev[t][1].record()
        if check:
            dues.append(n)
            checks.append(t)
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev]
    plain = sorted(m for t, m in enumerate(ms) if t not in checks)
    total = sum(ms)
    return {"steps": steps, "period": period, "layers": L, "capacity": cap,
            "ms_per_step": total / steps, "decode_step_ms": plain[len(plain) // 2],
            "check_step_ms": [ms[t] for t in checks], "due_per_check": dues,
            "tokens_per_s": B * steps / (total / 1e3), "status": K.read_status(status),
            "workload": "LaCache in the decode loop: batch 32, 4 layers, 28 query / 4 KV heads, "
                        "d=128, 4096-token contexts, S=2, O=1, rung 64, sink 64, recent 64, "
                        f"budget {budget} per layer, capacity {cap}, check every {period} steps"}


def gpu_arm(args, rank: int, world: int, local_rank: int) -> dict | None:
    import torch.distributed as dist
    from decode_kv_cache_kara_b200 import kara as K
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = WORKLOAD
    seed = rank_seed(rank)
    cache = synth.make_cache(wl, seed, dev)
    work = algorithmic_work(wl, cache)
    step = Step(cache, wl)
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    if K.read_status(step.status) != 0:
        raise RuntimeError(f"device status after warm-up: {K.status_str(K.read_status(step.status))}")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = K.kara_launch_count()
    t0.record()
    for i in range(args.steps):
        step.run(ev[i])
    t1.record()
    launches = K.kara_launch_count() - launches0
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = t0.elapsed_time(t1)
    if K.read_status(step.status) != 0:
        raise RuntimeError(f"device status: {K.status_str(K.read_status(step.status))}")

    op_ms = {"kara_score": [], "select+token2chunk": [], "kara_compact": [],
             "paged_decode_attn": []}
    for e in ev:
        op_ms["kara_score"].append(e[0].elapsed_time(e[1]))
        op_ms["select+token2chunk"].append(e[1].elapsed_time(e[2]))
        op_ms["kara_compact"].append(e[2].elapsed_time(e[3]))
        op_ms["paged_decode_attn"].append(e[3].elapsed_time(e[4]))
    avg = {k: sum(v) / len(v) for k, v in op_ms.items()}

    total_ms = max_over_ranks(total_ms, dev, world)
    ms_step = total_ms / args.steps
    tokens_step = wl.batch * wl.window * world
    value = whole_job_value(wl.batch * wl.window, world, ms_step)

    e2e = e2e_run(cache, wl, steps=min(args.steps, args.e2e_steps), warmup=2)
    e2e_ms = max_over_ranks(e2e["ms_per_step"], dev, world)
    if rank != 0:
        return None

    peaks, src = load_peaks()
    # the exponentials bound scoring: one per softmax element, 16 per clock per SM on the SFU
    n_exp = wl.window * wl.window * wl.hq * wl.batch
    sfu_floor_ms = n_exp / (16 * 148 * 1.965e9) * 1e3
    if step.score_fused:
        score_exec, score_note = 1.25, ("fused single-exponential kernel: S over 144 key rows "
                                        "per 128 owned keys (x1.125) plus the P'^T W column-sum "
                                        "product (N = 16, x0.125): executed = 1.25 x useful")
    else:
        score_exec, score_note = 2.0, ("two UMMA passes (row log-sum-exp, then column sums): "
                                       "executed flops are twice the useful Q K^T")
    kernels = {
        "kara_score": {"ms": avg["kara_score"], "bound": "tensor",
                       "useful_tflops": work["score_flops"] / avg["kara_score"] / 1e9,
                       "executed_tflops": score_exec * work["score_flops"] / avg["kara_score"] / 1e9,
                       "note": score_note,
                       "exp2_count": n_exp,
                       "sfu_floor_ms": sfu_floor_ms,
                       "frac_of_sfu_floor": sfu_floor_ms / avg["kara_score"]},
        "select+token2chunk": {"ms": avg["select+token2chunk"], "bound": "latency"},
        "kara_compact": {"ms": avg["kara_compact"], "bound": "hbm",
                         "gbs": work["compact_bytes"] / avg["kara_compact"] / 1e6},
        "paged_decode_attn": {"ms": avg["paged_decode_attn"], "bound": "hbm",
                              "gbs": work["decode_bytes"] / avg["paged_decode_attn"] / 1e6},
    }
    for k, v in kernels.items():
        if v["bound"] == "hbm":
            v["frac_of_hbm_" + src] = v["gbs"] / peaks["hbm_gbs"]
        elif v["bound"] == "tensor":
            v["frac_of_bf16_" + src] = v["useful_tflops"] / peaks["bf16_tflops"]
    dom = max((k for k in kernels if kernels[k]["bound"] in ("tensor", "hbm")),
              key=lambda k: kernels[k]["ms"])
    dk = kernels[dom]
    traffic = captured_traffic(dom)
    if dk["bound"] == "tensor":
        roof = {"kernel": dom, "bound": "tensor", "achieved": dk["useful_tflops"],
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": dk["useful_tflops"] / peaks["bf16_tflops"], "traffic": traffic,
                "peak_source": f"{src} bf16 burst (MEASURED_PEAKS.json bf16_tflops)"}
    else:
        roof = {"kernel": dom, "bound": "hbm", "achieved": dk["gbs"], "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": dk["gbs"] / peaks["hbm_gbs"], "traffic": traffic,
                "peak_source": f"{src} HBM copy (MEASURED_PEAKS.json hbm_gbs)"}

    if world == 1 and not args.no_lacache:
        lac = lacache_run(dev, args.lacache_batch)
        lac["frac_of_hbm_" + src] = lac["gbs"] / peaks["hbm_gbs"]
        kernels["lacache_compact"] = lac
    if world == 1 and not args.no_loop:
        kernels["decode_loop"] = decode_loop_run(dev)
        kernels["lacache_loop"] = lacache_loop_run(dev)
        kernels["variants"] = variants_run(step)

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(seed)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC, "batch_per_gpu": wl.batch, "layers": wl.layers,
                   "q_heads": wl.hq, "kv_heads": wl.hkv, "head_dim": wl.head_dim,
                   "context": wl.ctx_lo, "window": wl.window, "keep": wl.keep, "page": wl.page,
                   "anchor_frac": wl.anchor_frac, "gap_limit": wl.gap_limit, "widen": wl.widen,
                   "parallelism": f"dp{world} (independent sequences per rank)",
                   "l2": "inputs larger than L2 (window queries 235 MB, KV pool 302 MB per GPU)"},
        "roofline": roof,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": {"value": tokens_step / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                "d2h_bytes_per_step": e2e["d2h_bytes_per_step"], "ms_per_step": e2e_ms},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    return line


def cpu_baseline(seed: int, target_s: float = 15.0) -> dict:
    """The oracle as it stands on the host cores, on a bounded sample of the same workload:
    as many (sequence, KV head) units as take about target_s seconds (at most 256)."""
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    cache_cpu = synth.make_cache(WORKLOAD, seed, "cpu")
    dt, tokens = time_cpu_oracle_sample(cache_cpu, WORKLOAD, units=1, seed=seed)
    units = max(1, int(target_s / max(dt, 1e-3)))
    units = min(units, 256)
    dt, tokens = time_cpu_oracle_sample(cache_cpu, WORKLOAD, units=units, seed=seed + 1)
    return {"value": tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{units} (sequence, KV head) units of the layer workload: window scoring "
                      f"of its 7 query heads, top-k, Token2Chunk, compaction of its rows and "
                      f"decode of its 7 query heads; tokens counted as W/Hkv per unit",
            "seconds": dt}


def reference_arm(args, rank: int) -> dict | None:
    if rank != 0:
        return None
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    wl = WORKLOAD
    cache_cpu = synth.make_cache(wl, rank_seed(0), "cpu")
    for i in range(args.warmup):
        time_cpu_oracle_sample(cache_cpu, wl, units=1, seed=i)
    total, tokens = 0.0, 0.0
    for i in range(args.steps):
        dt, tk = time_cpu_oracle_sample(cache_cpu, wl, units=1, seed=10_000 + i)
        total += dt
        tokens += tk
    value = tokens / total
    sample = ("each step: one (sequence, KV head) unit of the layer workload through the fp64 "
              "oracle (scoring of 7 query heads x 1024 x 1024, top-k, Token2Chunk, compaction, "
              "decode); tokens counted as W/Hkv per unit")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC, "batch_per_gpu": wl.batch, "window": wl.window,
                   "keep": wl.keep, "parallelism": "host cores (oracle)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kara", "reference"], default="kara")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-lacache", action="store_true",
                    help="skip the LaCache ladder-compaction measurement (1 GPU only)")
    ap.add_argument("--lacache-batch", type=int, default=8)
    ap.add_argument("--no-loop", action="store_true",
                    help="skip the decode-loop measurement (kernels.decode_loop)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = reference_arm(args, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = gpu_arm(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
