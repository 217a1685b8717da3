"""Shared test helpers: device moves, numpy views for the oracle, tolerance checks."""

from __future__ import annotations

import numpy as np
import torch

from decode_kv_cache_kara_b200 import synth


def to_device(cache: dict, device="cuda") -> dict:
    out = dict(cache)
    for key in ("k", "v", "q_win"):
        if key in cache:
            out[key] = [t.to(device) for t in cache[key]]
    for key in ("block_table", "ctx_len", "free_list", "free_top", "q_dec"):
        if key in cache:
            out[key] = cache[key].to(device)
    return out


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy()


def i32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.int64)


def assert_scores_close(gpu: np.ndarray, ref: np.ndarray, rtol=1e-3, atol=1e-6):
    """The score tolerance: |gpu - ref| <= rtol*|ref| + atol elementwise."""
    err = np.abs(gpu - ref)
    bound = rtol * np.abs(ref) + atol
    bad = err > bound
    assert not bad.any(), (f"{int(bad.sum())} scores outside tolerance; worst rel "
                           f"{float((err / np.maximum(np.abs(ref), 1e-30)).max()):.3e}")


def assert_selection_matches(sel_gpu: np.ndarray, sel_ref: np.ndarray, ref_scores: np.ndarray,
                             rel=1e-3):
    """Kept-index sets equal except at near-ties: every index in one set but not the other
    has an oracle score within `rel` (relative) of the oracle's k-th largest score."""
    rows = sel_gpu.reshape(-1, sel_gpu.shape[-1])
    refs = sel_ref.reshape(-1, sel_ref.shape[-1])
    scs = ref_scores.reshape(-1, ref_scores.shape[-1])
    for a, b, s in zip(rows, refs, scs):
        diff = set(a.tolist()) ^ set(b.tolist())
        if not diff:
            continue
        kth = np.sort(s)[::-1][len(b) - 1]
        for j in diff:
            assert abs(s[j] - kth) <= rel * max(abs(kth), abs(s[j])), (j, s[j], kth)


def logical_rows(pool_bits: np.ndarray, table_row: np.ndarray, n: int, page: int = 16):
    slots = np.arange(n)
    return pool_bits[table_row[slots // page], slots % page]


def make(wl: synth.Workload, seed: int, device="cuda", layers=None):
    """Generate a cache on the CPU (small cases) and move it to the device."""
    cpu = synth.make_cache(wl, seed, "cpu", layers=layers)
    return cpu, to_device(cpu, device)
