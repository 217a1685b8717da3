"""Throughput benchmark of the Kara decode-time compression step on B200.

One step = one pass of the whole hot path over the "step" workload: a 28-layer 7B-class model
(28 query / 4 KV heads, d = 128) with a batch of 128 sequences whose paged caches hold ragged
contexts of 2K-16K tokens (page 16, so windows start at unaligned slots), every sequence due
(the worst-case check step of the 100-step schedule), window W = 1024, keep 204 (20 %),
Token2Chunk anchors 50 % / gap 8 / widen 1:

    kara_score per layer -> one kara_select_chunks over the rows of all layers -> one
    kara_compact over all layers -> paged_decode_attn per layer over the compressed cache

then the block table, lengths and free list are restored, so that every step sees the same
input (compaction writes only fresh blocks, so the old rows are still in place). Metric:
compressed KV tokens per second (window tokens of all due sequences / step time), whole job
over all ranks. Beside it, in `kernels`: the amortised cost under the 100-step schedule
(the decode loop with the tail-W trigger on the same shapes), the one-layer workload
(batch 32, 4096-token caches), the LaCache workload's three iterative ladder passes and the
score / selection variants.

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
WORKLOAD = synth.WORKLOADS["step"]
WORKLOAD_INDEX = 2            # its position among the five workloads (seed 1234 + index)
LAYER_WORKLOAD = synth.WORKLOADS["layer"]
WORKLOAD_DESC = ("step: 28-layer 7B-class model (28 query / 4 KV heads, head_dim 128), batch "
                 "128, ragged contexts uniform in [2048, 16384] tokens in 16-token pages, "
                 "window W=1024 (the last 1024 tokens), keep 204 (20%), Token2Chunk anchors 50% "
                 "/ gap 8 / widen 1, every sequence due (the worst-case check step of the "
                 "100-step schedule); score and select per layer, one compaction of all 28 "
                 "layers, then paged GQA decode of every layer over the compressed cache")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def bench_config(wl: synth.Workload, world: int) -> dict:
    """The `config` of both arms' JSON lines (the same workload, so the same dict)."""
    return {"workload": WORKLOAD_DESC, "batch_per_gpu": wl.batch, "layers": wl.layers,
            "q_heads": wl.hq, "kv_heads": wl.hkv, "head_dim": wl.head_dim,
            "context": [wl.ctx_lo, wl.ctx_hi], "window": wl.window, "keep": wl.keep,
            "page": wl.page, "anchor_frac": wl.anchor_frac, "gap_limit": wl.gap_limit,
            "widen": wl.widen, "due_per_step": wl.batch,
            "parallelism": f"dp{world} (independent sequences per rank)",
            "l2": "inputs larger than L2 (window queries 26.3 GB, KV pools about 70 GB per GPU)"}


def captured_traffic(op: str, workload: str):
    """DRAM bytes per launch of `op` from the committed ncu summary (profiles/traffic.txt),
    captured on a launch of `workload`'s shape; None when there is no such capture or the
    kernel source changed since (its sha256 no longer matches)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        parts = line.split()
        if len(parts) != 5 or line.startswith("#") or parts[0] != op or parts[4] != workload:
            continue
        src = os.path.join(ROOT, "decode_kv_cache_kara_b200", parts[1])
        if not os.path.exists(src):
            return None
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return int(parts[3]) if digest == parts[2] else None
    return None


def rank_seed(rank: int, index: int = WORKLOAD_INDEX) -> int:
    """Seed of a rank's batch: the workload's seed (1234 + its index), offset per rank so that
    every rank compresses its own, independent sequences."""
    return 1234 + index + 1000 * rank


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


def host_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


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
def decode_queries(cache: dict) -> list:
    """One decode query [B, Hq, d] per layer: the cache's own for layer 0, seeded N(0, 1) draws
    for the others."""
    q0 = cache["q_dec"]
    gen = torch.Generator(device=q0.device)
    gen.manual_seed(cache["seed"] + 77)
    out = [q0]
    for _ in range(1, len(cache["k"])):
        out.append(torch.randn(q0.shape, generator=gen, device=q0.device).to(q0.dtype))
    return out


class Step:
    """One compression step of the whole path, over every layer of a device-resident cache:
    scores of every layer, selection + Token2Chunk of every layer, one compaction of all
    layers, decode of every layer over the compressed cache."""

    OPS = ("kara_score", "select+token2chunk", "kara_compact", "paged_decode_attn")

    def __init__(self, cache: dict, wl: synth.Workload):
        from decode_kv_cache_kara_b200 import kara as K
        self.K = K
        self.wl = wl
        self.c = cache
        dev = cache["k"][0].device
        L = len(cache["k"])
        self.L = L
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
        self.q_dec = decode_queries(cache)
        self.scores = torch.empty((L, r, wl.hkv, wl.window), dtype=torch.float32, device=dev)
        self.sel = torch.empty((L, r, wl.hkv, wl.keep), dtype=torch.int32, device=dev)
        self.keep = torch.empty((L, r, wl.hkv, wl.keep), dtype=torch.int32, device=dev)
        self.out = torch.empty((L, wl.batch, hq, wl.head_dim), dtype=torch.bfloat16, device=dev)
        ws = max(K.kara_workspace_bytes(K.OP_SCORE, self.pool, r, wl.window, hq),
                 K.kara_workspace_bytes(K.OP_COMPACT, self.pool, r, wl.window, 0, wl.keep),
                 K.kara_workspace_bytes(K.OP_DECODE, self.pool, 0, 0, hq, 0))
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        # scoring: the fused cluster kernel for windows of up to 1024 keys and of 2048 (plus
        # the split-item sum when a cluster range ends inside an item, and the one-kernel
        # two-pass helper on the SMs the clusters leave idle when there are items enough),
        # else the three two-pass kernels; select + Token2Chunk in one kernel; compaction
        # check + plan + gather; decode stream + combine. One call's launches are recorded.
        n0 = K.kara_launch_count()
        K.kara_score(cache["q_win"][0], cache["k"][0], self.pool, wl.window,
                     scores=self.scores[0], workspace=self.ws, status=self.status)
        torch.cuda.synchronize()
        self.score_launches = K.kara_launch_count() - n0
        self.score_fused = wl.window <= 1024 or wl.window == 2048

    def restore(self):
        self.book.copy_(self.saved_book, non_blocking=True)

    def run(self, events=None, restore=True, layer_ready=None, layer_scored=None):
        """One step on the current stream. `layer_ready[l]`, if given, is an event the scoring
        of layer l waits for (its window queries copied in); `layer_scored[l]` is recorded
        once layer l is scored (its window-query buffer may then be overwritten)."""
        K, wl, c = self.K, self.wl, self.c
        rec = (lambda i: events[i].record()) if events is not None else (lambda i: None)
        rec(0)
        for layer in range(self.L):
            if layer_ready is not None:
                torch.cuda.current_stream().wait_event(layer_ready[layer])
            K.kara_score(c["q_win"][layer], c["k"][layer], self.pool, wl.window,
                         scores=self.scores[layer], workspace=self.ws, status=self.status)
            if layer_scored is not None:
                layer_scored[layer].record()
        rec(1)
        # selection and Token2Chunk are per (sequence, KV head) row: one launch over the rows
        # of every layer
        K.kara_select_chunks(self.scores, wl.keep, wl.anchor_frac, wl.gap_limit, wl.widen,
                             keep=self.keep, sel=self.sel)
        rec(2)
        K.kara_compact(c["k"], c["v"], self.pool, wl.window, self.keep, workspace=self.ws,
                       status=self.status)
        rec(3)
        for layer in range(self.L):
            K.paged_decode_attn(self.q_dec[layer], c["k"][layer], c["v"][layer], self.pool,
                                out=self.out[layer], workspace=self.ws, status=self.status)
        rec(4)
        if restore:
            self.restore()


def algorithmic_work(wl: synth.Workload, cache: dict) -> dict:
    """Algorithmic flops / bytes of each op over one step (all layers; inputs before the
    step). Scoring: one Q K^T per (sequence, layer). Compaction: the K and V head-rows moved
    (the prefix rows of the first window page and the k kept rows per KV head), read and
    written. Decode: the K and V rows of the compressed contexts, plus q and out."""
    L = len(cache["k"])
    ctx = cache["ctx_len"].cpu().numpy().astype(np.int64)
    r, W, d, hq, hkv, k = wl.batch, wl.window, wl.head_dim, wl.hq, wl.hkv, wl.keep
    score_flops = 2.0 * W * W * d * hq * r * L
    off = (ctx - W) % wl.page
    rows = (hkv * (k + off)).sum()                               # head-rows per layer
    compact_bytes = float(rows * d * 2 * 2 * 2 * L)              # K and V, read + write
    n_after = ctx - W + k
    decode_bytes = float((n_after.sum() * hkv * d * 2 * 2 + 2 * r * hq * d * 2) * L)
    return {"score_flops": score_flops, "compact_bytes": compact_bytes,
            "decode_bytes": decode_bytes}


def time_step(step: Step, steps: int, warmup: int, world: int = 1, sampler=None):
    """Warm-up, then `steps` timed steps between a barrier and a synchronize on both sides.
    Returns (total ms, per-op average ms, launches in the timed region, clocks)."""
    K = step.K
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    if K.read_status(step.status) != 0:
        raise RuntimeError(f"device status after warm-up: {K.status_str(K.read_status(step.status))}")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sampler is not None:
        sampler.start()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = K.kara_launch_count()
    t0.record()
    for i in range(steps):
        step.run(ev[i])
    t1.record()
    launches = K.kara_launch_count() - launches0
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    clocks = sampler.stop() if sampler is not None else None
    if K.read_status(step.status) != 0:
        raise RuntimeError(f"device status: {K.status_str(K.read_status(step.status))}")
    avg = {}
    for j, name in enumerate(Step.OPS):
        avg[name] = sum(e[j].elapsed_time(e[j + 1]) for e in ev) / steps
    return t0.elapsed_time(t1), avg, launches, clocks


def kernel_entries(wl: synth.Workload, work: dict, avg: dict, step: Step, peaks: dict,
                   src: str) -> dict:
    """Per-op times of a step and their fractions of the measured peaks."""
    L = step.L
    n_exp = wl.window * wl.window * wl.hq * wl.batch * L
    sfu_floor_ms = n_exp / (16 * 148 * 1.965e9) * 1e3
    if step.score_fused:
        score_exec, score_note = None, ("fused single-exponential kernel (executed = 1.125 x "
                                        "useful: S over the 128 owned keys plus the P'^T W "
                                        "column-sum product, N = 16), and beside it, on the SMs "
                                        "its clusters leave idle, the one-kernel two-pass helper "
                                        "for a few percent of the items (executed 2 x useful) "
                                        "when the batch is large enough")
    else:
        score_exec, score_note = 2.0, ("two UMMA passes (row log-sum-exp, then column sums): "
                                       "executed flops are twice the useful Q K^T")
    ms_score = avg["kara_score"]
    kernels = {
        "kara_score": {"ms": ms_score, "bound": "tensor", "launches_of_op": L,
                       "useful_tflops": work["score_flops"] / ms_score / 1e9,
                       "executed_tflops": (score_exec * work["score_flops"] / ms_score / 1e9
                                           if score_exec is not None else None),
                       "launches_per_call": step.score_launches,
                       "note": score_note, "exp2_count": n_exp, "sfu_floor_ms": sfu_floor_ms,
                       "frac_of_sfu_floor": sfu_floor_ms / ms_score},
        "select+token2chunk": {"ms": avg["select+token2chunk"], "bound": "latency",
                               "launches_of_op": 1},
        "kara_compact": {"ms": avg["kara_compact"], "bound": "hbm", "launches_of_op": 1,
                         "gbs": work["compact_bytes"] / avg["kara_compact"] / 1e6,
                         "bytes": work["compact_bytes"]},
        "paged_decode_attn": {"ms": avg["paged_decode_attn"], "bound": "hbm", "launches_of_op": L,
                              "gbs": work["decode_bytes"] / avg["paged_decode_attn"] / 1e6,
                              "bytes": work["decode_bytes"]},
    }
    for v in kernels.values():
        if v["bound"] == "hbm":
            v["frac_of_hbm_" + src] = v["gbs"] / peaks["hbm_gbs"]
        elif v["bound"] == "tensor":
            v["frac_of_bf16_" + src] = v["useful_tflops"] / peaks["bf16_tflops"]
            v["frac_of_bf16_sustained_" + src] = v["useful_tflops"] / peaks.get(
                "bf16_tflops_sustained", peaks["bf16_tflops"])
    return kernels


def roofline_entry(kernels: dict, peaks: dict, src: str, total_ms: float, clocks,
                   traffic_of) -> dict:
    """The bench line's `roofline`: the dominant kernel (the longest op bound by the tensor
    pipe or by HBM), its achieved rate over its summed launch time and the measured peak it is
    held against. A tensor-bound kernel timed inside a long run (a timed region of a second or
    more, or with sw_power_cap seen in the clock samples) is held against the sustained bf16
    figure, one timed alone against the burst figure; both fractions are reported."""
    dom = max((k for k in kernels if kernels[k]["bound"] in ("tensor", "hbm")),
              key=lambda k: kernels[k]["ms"])
    dk = kernels[dom]
    traffic = traffic_of(dom)
    per_launch = (f"the op runs as {dk['launches_of_op']} launches per step (one per layer); "
                  "achieved = useful work of all of them / their summed duration")
    if dk["bound"] == "hbm":
        return {"kernel": dom, "bound": "hbm", "achieved": dk["gbs"], "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": dk["gbs"] / peaks["hbm_gbs"], "traffic": traffic,
                "peak_source": f"{src} HBM copy (MEASURED_PEAKS.json hbm_gbs)",
                "per_launch": per_launch}
    timed_s = total_ms / 1e3
    capped = bool(clocks) and "sw_power_cap" in (clocks.get("reasons") or [])
    sustained = timed_s >= 1.0 or capped
    sus_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    peak = sus_peak if sustained else peaks["bf16_tflops"]
    if sustained:
        source = (f"{src} bf16 sustained (MEASURED_PEAKS.json bf16_tflops_sustained): timed "
                  f"region {timed_s:.2f} s{', sw_power_cap active' if capped else ''}")
    else:
        source = (f"{src} bf16 burst (MEASURED_PEAKS.json bf16_tflops): timed region "
                  f"{timed_s:.2f} s, no power cap seen")
    return {"kernel": dom, "bound": "tensor", "achieved": dk["useful_tflops"], "peak": peak,
            "unit": "TFLOP/s", "frac": dk["useful_tflops"] / peak, "traffic": traffic,
            "frac_of_burst": dk["useful_tflops"] / peaks["bf16_tflops"],
            "frac_of_sustained": dk["useful_tflops"] / sus_peak,
            "peak_source": source, "per_launch": per_launch}


def time_cpu_oracle_sample(cache_cpu: dict, wl: synth.Workload, units: int = 1, seed: int = 0,
                           layers_per_step: int = 1):
    """The oracle as it stands on `units` (sequence, KV head) units of one layer of a CPU
    cache: score (the unit's G query heads), select, Token2Chunk, compaction of its rows,
    decode of its G query heads over the compressed sequence. Returns (seconds, tokens):
    a unit is W / (Hkv * layers_per_step) window tokens of a step that compresses
    `layers_per_step` layers."""
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
    return dt, units * wl.window / (wl.hkv * layers_per_step)


def oracle_sample_cache(seed: int) -> dict:
    """A CPU cache with the step workload's shapes and value recipe (four sequences, one
    layer), for timing the oracle on units of the same workload."""
    return synth.make_cache(WORKLOAD.with_(batch=4, layers=1), seed, "cpu")


def e2e_run(step: Step, steps: int, warmup: int, world: int = 1) -> dict:
    """The same step through the public API with HOST inputs: every step copies the window
    queries of every layer, the decode queries and the pool bookkeeping from pinned host
    memory into the step's device buffers, runs the step and reads back every layer's decode
    output, the keep sets, the block table and the lengths. The KV pools are the serving
    engine's device-resident cache (state kept across steps, not an input of one step).
    The window queries (26 GB a step) move layer by layer on a copy stream: scoring of a
    layer waits for its copy, and the next step's copy of a layer waits until this step has
    scored it, so copies overlap the compute of the layers before them. The timed region
    starts before the first step's copies and ends after the last step's read-back.
    With several ranks on one host (about 200 GB of host memory on the benchmark machine),
    one pinned layer of window queries serves as every layer's host input, so that a rank
    pins 1 GB rather than 26 GB; the bytes copied per step are the same."""
    c = step.c
    comp = torch.cuda.current_stream()
    copy_s = torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in c["q_win"]]
    scored = [torch.cuda.Event() for _ in c["q_win"]]

    def pinned_copy(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    if world == 1:
        host_q = [pinned_copy(t) for t in c["q_win"]]
    else:
        host_q = [pinned_copy(c["q_win"][0])] * len(c["q_win"])
    host_qd = [pinned_copy(t) for t in step.q_dec]
    host_book = pinned_copy(step.saved_book)
    out_host = {"out": torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory(),
                "keep": torch.empty(step.keep.shape, dtype=torch.int32).pin_memory(),
                "block_table": torch.empty(c["block_table"].shape, dtype=torch.int32).pin_memory(),
                "ctx_len": torch.empty(c["ctx_len"].shape, dtype=torch.int32).pin_memory()}
    h2d_bytes = sum(t.numel() * t.element_size() for t in host_q + host_qd + [host_book])
    d2h_bytes = sum(t.numel() * t.element_size() for t in out_host.values())

    def one():
        with torch.cuda.stream(copy_s):
            for layer, (d_, h_) in enumerate(zip(c["q_win"], host_q)):
                copy_s.wait_event(scored[layer])     # the previous step has scored the layer
                d_.copy_(h_, non_blocking=True)
                copied[layer].record(copy_s)
        for d_, h_ in zip(step.q_dec, host_qd):
            d_.copy_(h_, non_blocking=True)
        step.book.copy_(host_book, non_blocking=True)   # the step's bookkeeping from the host
        step.run(restore=False, layer_ready=copied, layer_scored=scored)
        out_host["out"].copy_(step.out, non_blocking=True)
        out_host["keep"].copy_(step.keep, non_blocking=True)
        out_host["block_table"].copy_(c["block_table"], non_blocking=True)
        out_host["ctx_len"].copy_(c["ctx_len"], non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    copy_s.wait_event(e0)                            # no copy of the timed steps starts earlier
    for _ in range(steps):
        one()
    e1.record(comp)
    torch.cuda.synchronize()
    step.restore()
    ms = e0.elapsed_time(e1) / steps
    del host_q, host_qd
    return {"ms_per_step": ms, "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes}


def layer_workload_run(dev, steps: int, warmup: int, peaks: dict, src: str) -> dict:
    """The one-layer workload (batch 32, 28 query / 4 KV heads, 4096-token caches, W=1024,
    keep 204) through the same step, for comparison with the per-layer numbers."""
    wl = LAYER_WORKLOAD
    cache = synth.make_cache(wl, 1234 + 1, dev)
    step = Step(cache, wl)
    work = algorithmic_work(wl, cache)
    total, avg, launches, _ = time_step(step, steps, warmup)
    out = {"workload": "layer: one 7B-class layer, batch 32, 28 query / 4 KV heads, d=128, "
                       "4096-token caches, W=1024, keep 204",
           "ms_per_step": total / steps,
           "tokens_per_s": wl.batch * wl.window / (total / steps / 1e3),
           "gpu_launches_per_step": launches / steps,
           "kernels": kernel_entries(wl, work, avg, step, peaks, src)}
    out["variants"] = variants_run(step)
    del step, cache
    torch.cuda.empty_cache()
    return out


def lacache_run(dev, batch: int, peaks: dict, src: str) -> dict:
    """The LaCache workload's three iterative ladder passes (batch 8, 32 layers, 8 KV heads,
    64K-token caches, S=8, O=4, rung 64, budget 8192 per layer): pass 1 keeps 8192 slots per
    layer of the full cache (the oldest 32768 slots are dropped in every layer), then 24576
    new tokens are appended to every sequence (untimed: blocks popped from the free list,
    their K/V drawn from N(0, 1)), refilling the cache to its capacity, and the ladder runs
    again; passes 2 and 3 compress pass 1's survivors further. Each pass is timed with CUDA
    events. A warm-up pass runs first and its bookkeeping is restored."""
    from decode_kv_cache_kara_b200 import kara as K
    wl = synth.WORKLOADS["lacache"].with_(batch=batch)
    ex = wl.extra
    cache = synth.make_cache(wl, 1234 + 4, dev, with_queries=False)
    pool = K.PagedPool.from_cache(cache)
    saved = {k: cache[k].clone() for k in ("block_table", "ctx_len", "free_list", "free_top")}
    ws = torch.empty(K.kara_workspace_bytes(K.OP_LACACHE, pool, wl.batch, 0, 0, ex["budget"]),
                     dtype=torch.uint8, device=dev)
    status = K.new_status(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + 9)

    def one():
        K.lacache_compact(cache["k"], cache["v"], pool, ex["span"], ex["overlap"], ex["rung"],
                          ex["budget"], ex["sink"], ex["recent"], workspace=ws, status=status)

    def refill(tokens: int):
        # append `tokens` slots to every sequence: their pages are popped from the free list
        # (stack top first, sequences in order), their K/V rows drawn from N(0, 1)
        pages = tokens // wl.page
        top = int(cache["free_top"][0])
        need = wl.batch * pages
        if need > top:
            raise RuntimeError("LaCache refill: free list too short")
        ids = cache["free_list"][top - need:top].flip(0).view(wl.batch, pages)
        p0 = cache["ctx_len"].long() // wl.page
        cols = p0[:, None] + torch.arange(pages, device=dev)[None, :]
        cache["block_table"].scatter_(1, cols, ids)
        cache["free_top"][0] = top - need
        cache["ctx_len"] += tokens
        flat = ids.reshape(-1).long()
        for layer in range(wl.layers):
            for pool_t in (cache["k"][layer], cache["v"][layer]):
                pool_t[flat] = torch.randn((flat.numel(),) + tuple(pool_t.shape[1:]),
                                           generator=gen, device=dev).to(pool_t.dtype)

    one()                                   # warm-up pass, then back to the full cache
    torch.cuda.synchronize()
    for k, t in saved.items():
        cache[k].copy_(t)
    passes = []
    for i in range(ex["passes"]):
        if i > 0:
            refill(ex["refill"])
        torch.cuda.synchronize()
        n_before = int(cache["ctx_len"][0])
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        one()
        e1.record()
        torch.cuda.synchronize()
        passes.append({"ms": e0.elapsed_time(e1), "ctx_before": n_before,
                       "ctx_after": int(cache["ctx_len"][0])})
    st = K.read_status(status)
    # every layer keeps `budget` slots: K and V rows of [Hkv, d] read once and written once
    nbytes = 2 * 2 * wl.batch * wl.layers * ex["budget"] * wl.hkv * wl.head_dim * 2
    for p in passes:
        p["gbs"] = nbytes / p["ms"] / 1e6
        p["frac_of_hbm_" + src] = p["gbs"] / peaks["hbm_gbs"]
    ms = sum(p["ms"] for p in passes) / len(passes)
    del cache, saved, ws
    torch.cuda.empty_cache()
    return {"ms": ms, "bound": "hbm", "gbs": nbytes / ms / 1e6, "bytes_per_pass": nbytes,
            "frac_of_hbm_" + src: nbytes / ms / 1e6 / peaks["hbm_gbs"], "passes": passes,
            "status": st,
            "workload": f"lacache: batch {wl.batch}, 32 layers, 8 KV heads, d=128, 64K-token "
                        f"caches, S=8, O=4, rung 64, budget 8192 per layer; three iterative "
                        f"passes (all layers each), 24576 tokens appended before passes 2 and 3"}


def gqa8b_run(dev, peaks: dict, src: str, steps: int = 5, warmup: int = 3) -> dict:
    """The 8B-GQA workload (32 query / 8 KV heads, d=128, batch 256, ragged contexts uniform in
    [8192, 32768], W=2048, keep 409), one layer: its 32 layers' KV pools (about 690 GB) do not
    fit on one GPU, so one layer's pool (about 21.5 GB, plus 4.3 GB of window queries) is
    resident, the per-layer step (score, select + Token2Chunk, compaction, decode) is timed like
    the headline step, and the 32-layer step is extrapolated as 32 x the per-layer time
    (labelled as such). Then block free and reuse: W new tokens are appended to every sequence
    (untimed; their pages popped from the free list, so they reuse blocks the first compaction
    freed) and a second compression over the new window is timed."""
    from decode_kv_cache_kara_b200 import kara as K
    wl = synth.WORKLOADS["gqa8b"].with_(layers=1)
    cache = synth.make_cache(wl, 1234 + 3, dev, extra_pages=wl.window // wl.page + 2)
    work = algorithmic_work(wl, cache)
    step = Step(cache, wl)
    total, avg, launches, _ = time_step(step, steps, warmup)
    per_layer = total / steps
    kernels = kernel_entries(wl, work, avg, step, peaks, src)
    # block free and reuse: compact once (kept), append W tokens, time the second compression
    step.run(restore=False)
    torch.cuda.synchronize()
    freed_top = int(cache["free_top"][0])
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + 13)
    pages = wl.window // wl.page
    n = cache["ctx_len"].long()
    first = (n + wl.page - 1) // wl.page            # first page the new tokens need
    last = (n + wl.window + wl.page - 1) // wl.page
    need = (last - first).cpu().tolist()
    top = freed_top
    table = cache["block_table"]
    for b in range(wl.batch):                        # pages popped from the stack top, in order
        cnt = need[b]
        ids = cache["free_list"][top - cnt:top].flip(0)
        table[b, int(first[b]):int(first[b]) + cnt] = ids
        top -= cnt
    cache["free_top"][0] = top
    slots = n[:, None] + torch.arange(wl.window, device=dev)[None, :]
    blk = torch.gather(table.long(), 1, slots // wl.page)
    for pool_t in (cache["k"][0], cache["v"][0]):
        pool_t[blk, slots % wl.page] = torch.randn((wl.batch, wl.window, wl.hkv, wl.head_dim),
                                                   generator=gen, device=dev).to(pool_t.dtype)
    cache["ctx_len"] += wl.window
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    K.kara_score(cache["q_win"][0], cache["k"][0], step.pool, wl.window, scores=step.scores[0],
                 workspace=step.ws, status=step.status)
    K.kara_select_chunks(step.scores[0], wl.keep, wl.anchor_frac, wl.gap_limit, wl.widen,
                         keep=step.keep[0])
    K.kara_compact(cache["k"], cache["v"], step.pool, wl.window, step.keep, workspace=step.ws,
                   status=step.status)
    e1.record()
    torch.cuda.synchronize()
    st = K.read_status(step.status)
    tokens = wl.batch * wl.window
    out = {"workload": "gqa8b: 8B-class GQA, 32 query / 8 KV heads, d=128, batch 256, ragged "
                       "contexts [8192, 32768], W=2048, keep 409; one layer resident, the "
                       "32-layer step extrapolated as 32 x the per-layer step",
           "per_layer_ms": per_layer,
           "step_ms_extrapolated_x32": 32 * per_layer,
           "tokens_per_s_extrapolated": tokens / (32 * per_layer / 1e3),
           "gpu_launches_per_layer_step": launches / steps,
           "kernels_per_layer": kernels,
           "second_compression_after_reuse_ms": e0.elapsed_time(e1),
           "second_compression_status": st,
           "note": "scoring at W=2048 takes the fused kernel on clusters of 16 CTAs (a "
                   "non-portable cluster size); the second compression pops blocks freed by the "
                   "first"}
    del step, cache
    torch.cuda.empty_cache()
    return out


def compress_compare(step: Step, reps: int = 5) -> dict:
    """The step's selection + Token2Chunk and compaction of all layers as the two calls it
    times (kara_select_chunks, kara_compact) against the fused kara_compress, on the step's
    own scores; the bookkeeping is restored before every run (not timed)."""
    K, wl, c = step.K, step.wl, step.c

    def timed(fn):
        out = []
        for _ in range(reps + 1):
            step.restore()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            out.append(e0.elapsed_time(e1))
        return sorted(out[1:])[reps // 2]

    def two_calls():
        K.kara_select_chunks(step.scores, wl.keep, wl.anchor_frac, wl.gap_limit, wl.widen,
                             keep=step.keep, sel=step.sel)
        K.kara_compact(c["k"], c["v"], step.pool, wl.window, step.keep, workspace=step.ws,
                       status=step.status)

    def fused():
        K.kara_compress(step.scores, c["k"], c["v"], step.pool, wl.window, wl.keep,
                        wl.anchor_frac, wl.gap_limit, wl.widen, keep=step.keep,
                        workspace=step.ws, status=step.status)

    res = {"select_chunks_then_compact_ms": timed(two_calls), "compress_ms": timed(fused)}
    step.restore()
    torch.cuda.synchronize()
    res["status"] = K.read_status(step.status)
    res["note"] = ("all 28 layers of the step workload from the step's scores; median of "
                   f"{reps} runs")
    return res


def variants_run(step, reps: int = 10) -> dict:
    """The score and selection variants on the one-layer workload (its window queries and
    cache, not changed by them): kara_score_ex with the mean and with the max aggregation, and
    the selection shared across KV heads (head sums, select, Token2Chunk, expansion to every
    head). Average times with CUDA events over `reps` calls after one untimed call."""
    K, wl, c = step.K, step.wl, step.c
    scores, keep, sel = step.scores[0], step.keep[0], step.sel[0]
    tot = torch.empty((wl.batch, wl.window), dtype=torch.float32, device=scores.device)
    shared = torch.empty((wl.batch, wl.keep), dtype=torch.int32, device=tot.device)
    sel_t = torch.empty((wl.batch, wl.keep), dtype=torch.int32, device=tot.device)

    def score(agg):
        K.kara_score_ex(c["q_win"][0], c["k"][0], step.pool, wl.window, agg=agg,
                        scores=scores, workspace=step.ws, status=step.status)

    def shared_select():
        K.kara_sum_heads(scores, out=tot)
        K.kara_select(tot, wl.keep, sel=sel_t)
        K.kara_token2chunk(tot, sel_t, wl.anchor_frac, wl.gap_limit, wl.widen, keep=shared)
        K.kara_expand_keep(shared, wl.hkv, keep=keep)

    out = {}

    def select_then_chunks():
        K.kara_select(scores, wl.keep, sel=sel)
        K.kara_token2chunk(scores, sel, wl.anchor_frac, wl.gap_limit, wl.widen, keep=keep)

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

    # selection, Token2Chunk and compaction: two calls against kara_compress (plan + one
    # fused kernel); the bookkeeping is restored between repetitions, untimed
    def compact_pair():
        K.kara_select_chunks(scores, wl.keep, wl.anchor_frac, wl.gap_limit, wl.widen, keep=keep)
        K.kara_compact(c["k"], c["v"], step.pool, wl.window, step.keep, workspace=step.ws,
                       status=step.status)

    def compress():
        K.kara_compress(step.scores, c["k"], c["v"], step.pool, wl.window, wl.keep,
                        wl.anchor_frac, wl.gap_limit, wl.widen, keep=step.keep,
                        workspace=step.ws, status=step.status)

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
    out["note"] = ("one-layer workload; max runs the fused kernel with a per-key column "
                   "maximum in place of the column-sum product; shared = head sums, one "
                   "select + Token2Chunk per (sequence, layer), "
                   "keep copied to the 4 KV heads; select_then_token2chunk = the two calls the "
                   "step's fused kara_select_chunks replaces")
    return out


def decode_loop_run(dev, wl: synth.Workload, seed: int, steps: int = 200, period: int = 100,
                    warm: int = 10) -> dict:
    """The amortised step under the 100-step schedule, on the bench workload's shapes (every
    layer): every decode step runs kara_step_begin, kara_decode_append per layer (the new
    token's attention, its K/V into the cache, its query into the layer's window-query ring)
    and kara_step_end; every `period` steps the sequences whose uncompressed tail reached W
    are due and are compressed (kara_score_ring and kara_select_chunks per layer, one
    kara_compact of all layers, kara_reset_tails). Tails start uniform over [0, W) and the
    rings hold N(0, 1) queries, as in the middle of a generation, so that each check finds
    about batch * period / W due sequences. Timed with CUDA events per step; a check step
    includes the host read of the due count that sizes its compression."""
    from decode_kv_cache_kara_b200 import kara as K
    W, B, L = wl.window, wl.batch, wl.layers
    cache = synth.make_cache(wl, seed, dev, with_queries=False,
                             extra_pages=(steps + warm) // wl.page + 2)
    pool = K.PagedPool.from_cache(cache)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed + 5)
    rings = [torch.randn((B, 2 * W, wl.hq, wl.head_dim), generator=gen, device=dev)
             .to(torch.bfloat16) for _ in range(L)]
    tail = torch.randint(0, W, (B,), generator=gen, device=dev, dtype=torch.int32)
    inputs = [[[torch.randn(shape, generator=gen, device=dev).to(torch.bfloat16)
                for shape in ((B, wl.hq, wl.head_dim), (B, wl.hkv, wl.head_dim),
                              (B, wl.hkv, wl.head_dim))] for _ in range(L)] for _ in range(4)]
    out = torch.empty((L, B, wl.hq, wl.head_dim), dtype=torch.bfloat16, device=dev)
    ws_dec = torch.empty(K.kara_workspace_bytes(K.OP_DECODE, pool, 0, 0, wl.hq, 0),
                         dtype=torch.uint8, device=dev)
    ws = torch.empty(max(K.kara_workspace_bytes(K.OP_SCORE, pool, B, W, wl.hq),
                         K.kara_workspace_bytes(K.OP_COMPACT, pool, B, W, 0, wl.keep)),
                     dtype=torch.uint8, device=dev)
    scores = torch.empty((L, B, wl.hkv, W), dtype=torch.float32, device=dev)
    keep = torch.empty((L, B, wl.hkv, wl.keep), dtype=torch.int32, device=dev)
    due = torch.zeros(B, dtype=torch.int32, device=dev)
    due_count = torch.zeros(1, dtype=torch.int32, device=dev)
    status = K.new_status(dev)

    def step(t, check):
        K.kara_step_begin(pool, status)
        for layer in range(L):
            q, kn, vn = inputs[t % len(inputs)][layer]
            K.kara_decode_append(q, kn, vn, cache["k"][layer], cache["v"][layer], pool,
                                 rings[layer], W, out=out[layer], workspace=ws_dec, status=status)
        K.kara_step_end(pool, tail, W, check, due, due_count)
        if not check:
            return 0
        cnt = int(due_count.item())
        if cnt:
            seq = due[:cnt]
            # the keep sets of the due sequences, [L, cnt, Hkv, k] contiguous
            kp = keep.view(-1)[:L * cnt * wl.hkv * wl.keep].view(L, cnt, wl.hkv, wl.keep)
            for layer in range(L):
                K.kara_score_ring(rings[layer], cache["k"][layer], pool, W, seq, cnt,
                                  scores=scores[layer, :cnt], workspace=ws, status=status)
                K.kara_select_chunks(scores[layer, :cnt], wl.keep, wl.anchor_frac, wl.gap_limit,
                                     wl.widen, keep=kp[layer])
            K.kara_compact(cache["k"], cache["v"], pool, W, kp, seq_ids=seq, workspace=ws,
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
    plain_ms = plain[len(plain) // 2]
    extra = [ms[t] - plain_ms for t in checks]
    comp_tokens = sum(dues) * W
    res = {"steps": steps, "period": period, "layers": L, "ms_per_step": total / steps,
           "decode_step_ms": plain_ms, "check_step_ms": [ms[t] for t in checks],
           "due_per_check": dues, "compression_ms_per_check": extra,
           "compressed_tokens_per_s": (comp_tokens / (sum(extra) / 1e3)
                                       if sum(extra) > 0 else None),
           "compression_share_of_time": sum(extra) / total,
           "decode_tokens_per_s": B * steps / (total / 1e3), "status": st,
           "workload": f"decode loop: batch {B}, {L} layers, 28 query / 4 KV heads, d=128, "
                       f"ragged contexts [{wl.ctx_lo}, {wl.ctx_hi}], W={W}, keep {wl.keep}, "
                       f"check every {period} steps (tail-W trigger), tails uniform over [0, W)"}
    del cache, rings, inputs
    torch.cuda.empty_cache()
    return res


def lacache_loop_run(dev, steps: int = 200, period: int = 100, warm: int = 10) -> dict:
    """LaCache inside the decode loop on the one-layer workload's shapes with 4 layers (batch
    32, 28 query / 4 KV heads, d=128, 4096-token contexts): every step kara_step_begin, one
    kara_decode_append per layer and kara_step_end with the capacity trigger; the ladder
    (S = 2, O = 1, rung 64, sink 64, recent 64, budget 2048 per layer, so capacity
    64 + 64 + 1920 * 4 / 2 = 3968 slots) runs on the sequences due at a check step. Timed with
    CUDA events per step; a check step includes the host read of the due count."""
    from decode_kv_cache_kara_b200 import kara as K
    wl = LAYER_WORKLOAD.with_(layers=4)
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
    res = {"steps": steps, "period": period, "layers": L, "capacity": cap,
           "ms_per_step": total / steps, "decode_step_ms": plain[len(plain) // 2],
           "check_step_ms": [ms[t] for t in checks], "due_per_check": dues,
           "tokens_per_s": B * steps / (total / 1e3), "status": K.read_status(status),
           "workload": "LaCache in the decode loop: batch 32, 4 layers, 28 query / 4 KV heads, "
                       "d=128, 4096-token contexts, S=2, O=1, rung 64, sink 64, recent 64, "
                       f"budget {budget} per layer, capacity {cap}, check every {period} steps"}
    del cache
    torch.cuda.empty_cache()
    return res


def gpu_arm(args, rank: int, world: int, local_rank: int) -> dict | None:
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = WORKLOAD if args.layers is None else WORKLOAD.with_(layers=args.layers)
    seed = rank_seed(rank)
    peaks, src = load_peaks()
    cache = synth.make_cache(wl, seed, dev)
    work = algorithmic_work(wl, cache)
    step = Step(cache, wl)
    sampler = ClockSampler(local_rank)
    total_ms, avg, launches, clocks = time_step(step, args.steps, args.warmup, world, sampler)
    total_ms = max_over_ranks(total_ms, dev, world)
    ms_step = total_ms / args.steps
    tokens_step = wl.batch * wl.window          # window tokens compressed per step and rank
    value = whole_job_value(tokens_step, world, ms_step)

    e2e = None
    if not args.no_e2e:
        e2e = e2e_run(step, steps=args.e2e_steps, warmup=1, world=world)
        e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], dev, world)
    kernels = kernel_entries(wl, work, avg, step, peaks, src)
    fused_compression = (compress_compare(step) if world == 1 and not args.no_layer else None)
    del step, cache
    torch.cuda.empty_cache()
    if rank != 0:
        return None

    roof = roofline_entry(kernels, peaks, src, total_ms, clocks,
                          lambda op: captured_traffic(op, wl.name))

    comp_ms = sum(kernels[op]["ms"] for op in ("kara_score", "select+token2chunk", "kara_compact"))
    kernels["compression_only"] = {
        "ms": comp_ms, "tokens_per_s": whole_job_value(tokens_step, world, comp_ms),
        "note": "the step without its decode: scoring, selection + Token2Chunk and compaction "
                "of all layers (per-op event times of the timed steps)"}
    if fused_compression is not None:
        kernels["fused_compression"] = fused_compression
    if world == 1 and not args.no_loop:
        kernels["amortised_100_step_schedule"] = decode_loop_run(dev, wl, seed + 50)
    if world == 1 and not args.no_layer:
        kernels["layer"] = layer_workload_run(dev, max(3, min(args.steps, 20)), 3, peaks, src)
    if world == 1 and not args.no_lacache:
        kernels["lacache_compact"] = lacache_run(dev, args.lacache_batch, peaks, src)
    if world == 1 and not args.no_gqa8b:
        kernels["gqa8b"] = gqa8b_run(dev, peaks, src)
    if world == 1 and not args.no_loop:
        kernels["lacache_loop"] = lacache_loop_run(dev)

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(seed)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(wl, world),
        "roofline": roof,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if e2e is not None:
        line["e2e"] = {"value": tokens_step * world / (e2e["ms_per_step"] / 1e3), "unit": UNIT,
                       "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                       "d2h_bytes_per_step": e2e["d2h_bytes_per_step"],
                       "ms_per_step": e2e["ms_per_step"],
                       "note": "window queries of every layer (with several ranks, one pinned "
                               "layer serves every layer's copy), decode queries and the pool "
                               "bookkeeping copied from pinned host memory every step (the "
                               "window queries layer by layer on a copy stream, overlapping "
                               "the scoring of earlier layers and the previous step); decode "
                               "outputs, keep sets, block table and lengths read back; the KV "
                               "pools stay resident on the device"}
    return line


def cpu_baseline(seed: int, target_s: float = 15.0) -> dict:
    """The oracle as it stands on the host cores, on a bounded sample of the same workload:
    as many (sequence, layer, KV head) units as take about target_s seconds (at most 256)."""
    cores = host_cores()
    cache_cpu = oracle_sample_cache(seed)
    wl = WORKLOAD.with_(batch=4, layers=1)
    time_cpu_oracle_sample(cache_cpu, wl, units=1, seed=seed, layers_per_step=WORKLOAD.layers)
    dt, tokens = time_cpu_oracle_sample(cache_cpu, wl, units=2, seed=seed + 7,
                                        layers_per_step=WORKLOAD.layers)
    units = max(1, int(target_s / max(dt / 2, 1e-3)))
    units = min(units, 256)
    dt, tokens = time_cpu_oracle_sample(cache_cpu, wl, units=units, seed=seed + 1,
                                        layers_per_step=WORKLOAD.layers)
    return {"value": tokens / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{units} (sequence, layer, KV head) units of the step workload (ragged "
                      f"contexts 2K-16K, W=1024, keep 204): window scoring of the unit's 7 query "
                      f"heads, top-k, Token2Chunk, compaction of its rows and decode of its 7 "
                      f"query heads; tokens counted as W / (Hkv * 28 layers) per unit",
            "seconds": dt}


def reference_arm(args, rank: int) -> dict | None:
    if rank != 0:
        return None
    cores = host_cores()
    wl = WORKLOAD.with_(batch=4, layers=1)
    cache_cpu = oracle_sample_cache(rank_seed(0))
    for i in range(args.warmup):
        time_cpu_oracle_sample(cache_cpu, wl, units=1, seed=i, layers_per_step=WORKLOAD.layers)
    total, tokens = 0.0, 0.0
    for i in range(args.steps):
        dt, tk = time_cpu_oracle_sample(cache_cpu, wl, units=1, seed=10_000 + i,
                                        layers_per_step=WORKLOAD.layers)
        total += dt
        tokens += tk
    value = tokens / total
    sample = ("each step: one (sequence, layer, KV head) unit of the step workload through the "
              "fp64 oracle (scoring of 7 query heads x 1024 x 1024, top-k, Token2Chunk, "
              "compaction, decode); tokens counted as W / (Hkv * 28 layers) per unit")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": bench_config(WORKLOAD, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kara", "reference"], default="kara")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-input measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-lacache", action="store_true",
                    help="skip the LaCache ladder-compaction measurement (1 GPU only)")
    ap.add_argument("--lacache-batch", type=int, default=8)
    ap.add_argument("--no-loop", action="store_true",
                    help="skip the decode-loop measurements (amortised schedule, LaCache loop)")
    ap.add_argument("--no-layer", action="store_true",
                    help="skip the one-layer workload and the variants")
    ap.add_argument("--no-gqa8b", action="store_true",
                    help="skip the 8B-GQA workload's per-layer measurement")
    ap.add_argument("--layers", type=int, default=None,
                    help="layers of the step workload (default: all 28); fewer layers keep a "
                         "profiler capture of one layer's launches small")
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
