"""Python binding of libkara (ctypes). Argument marshalling only: every step runs in the CUDA
library declared in include/kara.h. Torch provides device memory and the current stream.

The functions carry the C names:
    kara_score, kara_select, kara_token2chunk, kara_compact, paged_decode_attn,
    lacache_compact, kara_workspace_bytes
There is no CPU fallback: a missing library raises ``KaraLibraryError``.
"""

from __future__ import annotations

import ctypes
import math
import os
import re
from dataclasses import dataclass

import torch

from . import build as _build

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_OUT_OF_BLOCKS = 3
ERR_CUDA = 4
ERR_TIMEOUT = 5
ERR_WORKSPACE = 6
ERR_BAD_BLOCK = 7

OP_SCORE, OP_COMPACT, OP_DECODE, OP_LACACHE = 1, 2, 3, 4
TRIM_TOKEN, TRIM_CHUNK = 0, 1      # Token2Chunk's trim: token by token, or whole chunks first
MAX_LAYERS = 128


class KaraLibraryError(ImportError):
    """libkara.so is missing or cannot be loaded."""


class KaraError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        detail = ""
        if code == ERR_CUDA:
            detail = " [" + lib().kara_last_error().decode() + "]"
        super().__init__(f"{where}: {status_str(code)} ({code}){detail}")


class _LayerKV(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p)]


class _Pool(ctypes.Structure):
    _fields_ = [("block_table", ctypes.c_void_p), ("ctx_len", ctypes.c_void_p),
                ("free_list", ctypes.c_void_p), ("free_top", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32),
                ("num_blocks", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class _LacacheParams(ctypes.Structure):
    _fields_ = [("span", ctypes.c_int32), ("overlap", ctypes.c_int32), ("rung", ctypes.c_int32),
                ("budget", ctypes.c_int32), ("sink", ctypes.c_int32), ("recent", ctypes.c_int32)]


_LIB = None
_P = ctypes.c_void_p
_I = ctypes.c_int32
_F = ctypes.c_float
_Z = ctypes.c_size_t

_SIGNATURES = {
    "kara_score": ([_P, _P, ctypes.POINTER(_Pool), _P, _I, _I, _I, _F, _P, _P, _Z, _P, _P], _I),
    "kara_select": ([_P, _I, _I, _I, _P, _P], _I),
    "kara_token2chunk": ([_P, _P, _I, _I, _I, _F, _I, _I, _P, _P], _I),
    "kara_compact": ([ctypes.POINTER(_LayerKV), _I, ctypes.POINTER(_Pool), _P, _I, _I, _I, _P, _P,
                      _Z, _P, _P], _I),
    "kara_compact_noalloc": ([ctypes.POINTER(_LayerKV), _I, ctypes.POINTER(_Pool), _P, _I, _I, _I,
                              _P, _P, _P], _I),
    "paged_decode_attn": ([_P, _P, _P, ctypes.POINTER(_Pool), _I, _F, _P, _P, _Z, _P, _P], _I),
    "lacache_compact": ([ctypes.POINTER(_LayerKV), _I, ctypes.POINTER(_Pool), _P, _I,
                         ctypes.POINTER(_LacacheParams), _P, _Z, _P, _P], _I),
    "kara_workspace_bytes": ([_I, ctypes.POINTER(_Pool), _I, _I, _I, _I], _Z),
    "kara_status_str": ([_I], ctypes.c_char_p),
    "kara_version": ([], ctypes.c_char_p),
    "kara_last_error": ([], ctypes.c_char_p),
    "kara_launch_count": ([], ctypes.c_uint64),
    "kara_wait_probe": ([_I, _P, _P], _I),
    "kara_score_ring": ([_P, _P, ctypes.POINTER(_Pool), _P, _I, _I, _I, _F, _P, _P, _Z, _P, _P],
                        _I),
    "kara_decode_append": ([_P, _P, _P, _P, _P, ctypes.POINTER(_Pool), _I, _F, _P, _I, _P, _P, _Z,
                            _P, _P], _I),
    "kara_step_begin": ([ctypes.POINTER(_Pool), _P, _P], _I),
    "kara_step_end": ([ctypes.POINTER(_Pool), _P, _I, _I, _I, _P, _P, _P], _I),
    "kara_reset_tails": ([_P, _P, _I, _I, _P], _I),
    "kara_score_ex": ([_P, _I, _P, ctypes.POINTER(_Pool), _P, _I, _I, _I, _F, _I, _P, _P, _Z, _P,
                       _P], _I),
    "kara_sum_heads": ([_P, _I, _I, _I, _P, _P], _I),
    "kara_expand_keep": ([_P, _I, _I, _I, _P, _P], _I),
    "kara_select_chunks": ([_P, _I, _I, _I, _F, _I, _I, _P, _P, _P], _I),
    "kara_select_chunks_ex": ([_P, _I, _I, _I, _F, _I, _I, _I, _P, _P, _P], _I),
    "kara_token2chunk_ex": ([_P, _P, _I, _I, _I, _F, _I, _I, _I, _P, _P], _I),
    "kara_compress": ([_P, ctypes.POINTER(_LayerKV), _I, ctypes.POINTER(_Pool), _P, _I, _I, _I, _F,
                       _I, _I, _P, _P, _Z, _P, _P], _I),
}


def library_path() -> str:
    return _build.LIB


def lib():
    """The loaded libkara (loaded once). Raises KaraLibraryError when it is not built."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise KaraLibraryError(
                f"{path} is missing: build it with `python -m decode_kv_cache_kara_b200.build`")
        try:
            handle = ctypes.CDLL(path)
        except OSError as e:  # pragma: no cover - depends on the host
            raise KaraLibraryError(f"cannot load {path}: {e}") from e
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = handle
    return _LIB


def declared_symbols(header: str | None = None) -> list:
    """Function names declared in include/kara.h (used by the ABI tests)."""
    header = header or os.path.join(_build.INCLUDE, "kara.h")
    text = open(header).read()
    return re.findall(r"^\s*(?:kara_status|size_t|uint64_t|const char\*)\s+(\w+)\s*\(", text,
                      re.M)


def kara_launch_count() -> int:
    """Kernel launches the library has issued in this process (difference two readings)."""
    return int(lib().kara_launch_count())


def status_str(code: int) -> str:
    return lib().kara_status_str(int(code)).decode()


def _check(code: int, where: str):
    if code != OK:
        raise KaraError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _require(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


@dataclass
class PagedPool:
    """The shared block table, lengths and free list of a paged cache (device tensors)."""
    block_table: torch.Tensor   # int32 [B, max_blocks]
    ctx_len: torch.Tensor       # int32 [B]
    free_list: torch.Tensor     # int32 [num_blocks]
    free_top: torch.Tensor      # int32 [1]
    num_blocks: int
    num_kv_heads: int
    head_dim: int
    page_size: int = 16

    @classmethod
    def from_cache(cls, cache: dict) -> "PagedPool":
        k0 = cache["k"][0]
        return cls(cache["block_table"], cache["ctx_len"], cache["free_list"], cache["free_top"],
                   int(k0.shape[0]), int(k0.shape[2]), int(k0.shape[3]), int(k0.shape[1]))

    def c_struct(self) -> _Pool:
        for name in ("block_table", "ctx_len", "free_list", "free_top"):
            _require(getattr(self, name), torch.int32, name)
        b, mb = self.block_table.shape
        return _Pool(self.block_table.data_ptr(), self.ctx_len.data_ptr(),
                     self.free_list.data_ptr(), self.free_top.data_ptr(), int(b), int(mb),
                     int(self.num_blocks), int(self.page_size), int(self.num_kv_heads),
                     int(self.head_dim))


def new_status(device=None) -> torch.Tensor:
    """A zeroed device status word."""
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def read_status(status: torch.Tensor) -> int:
    """Synchronises with the status word's stream and returns its value."""
    return int(status.item())


def kara_workspace_bytes(op: int, pool: PagedPool | None = None, num_seqs: int = 0,
                         window: int = 0, num_q_heads: int = 0, k_or_budget: int = 0) -> int:
    ps = ctypes.byref(pool.c_struct()) if pool is not None else None
    return int(lib().kara_workspace_bytes(op, ps, num_seqs, window, num_q_heads, k_or_budget))


def _workspace(nbytes: int, device, workspace):
    """The caller's workspace (a contiguous CUDA uint8 tensor), or a new one of nbytes."""
    if workspace is not None:
        _require(workspace, torch.uint8, "workspace")
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _status(status, device):
    """The caller's status word (a CUDA int32 tensor), or a new zeroed one."""
    if status is None:
        return new_status(device)
    _require(status, torch.int32, "status")
    return status


def kara_score(q_win: torch.Tensor, k_cache: torch.Tensor, pool: PagedPool, window: int,
               scale: float | None = None, seq_ids: torch.Tensor | None = None,
               scores: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
               status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Window scores [R, Hkv, W] fp32 (see kara_score in include/kara.h)."""
    _require(q_win, torch.bfloat16, "q_win")
    _require(k_cache, torch.bfloat16, "k_cache")
    r, w, hq, d = q_win.shape
    if w != window:
        raise ValueError("q_win's second dimension must equal the window")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if scores is None:
        scores = torch.empty((r, pool.num_kv_heads, window), dtype=torch.float32,
                             device=q_win.device)
    _require(scores, torch.float32, "scores")
    if seq_ids is not None:
        _require(seq_ids, torch.int32, "seq_ids")
    status = _status(status, q_win.device)
    ps = pool.c_struct()
    nbytes = kara_workspace_bytes(OP_SCORE, pool, r, window, hq)
    ws = _workspace(nbytes, q_win.device, workspace)
    _check(lib().kara_score(_ptr(q_win), _ptr(k_cache), ctypes.byref(ps), _ptr(seq_ids), r,
                            window, hq, float(scale), _ptr(scores), _ptr(ws), ws.numel(),
                            _ptr(status), _stream(stream)), "kara_score")
    return scores


AGG_SUM, AGG_MEAN, AGG_MAX = 0, 1, 2


def kara_score_ex(q: torch.Tensor, k_cache: torch.Tensor, pool: PagedPool, window: int,
                  agg: int = AGG_SUM, ring: bool = False, seq_ids: torch.Tensor | None = None,
                  num_seqs: int | None = None, scale: float | None = None,
                  scores: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                  status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Window scores [R, Hkv, W] with the aggregation agg (AGG_SUM / AGG_MEAN / AGG_MAX), the
    queries from q_win [R, W, Hq, d] or, with ring=True, from the ring [B, 2W, Hq, d]."""
    _require(q, torch.bfloat16, "q")
    _require(k_cache, torch.bfloat16, "k_cache")
    rows, w2, hq, d = q.shape
    if w2 != (2 * window if ring else window):
        raise ValueError("q's second dimension must be the window (2 * window for a ring)")
    if num_seqs is None:
        num_seqs = int(seq_ids.numel()) if seq_ids is not None else rows
    if seq_ids is not None:
        _require(seq_ids, torch.int32, "seq_ids")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if scores is None:
        scores = torch.empty((num_seqs, pool.num_kv_heads, window), dtype=torch.float32,
                             device=q.device)
    _require(scores, torch.float32, "scores")
    status = _status(status, q.device)
    ps = pool.c_struct()
    ws = _workspace(kara_workspace_bytes(OP_SCORE, pool, num_seqs, window, hq), q.device,
                    workspace)
    _check(lib().kara_score_ex(_ptr(q), 1 if ring else 0, _ptr(k_cache), ctypes.byref(ps),
                               _ptr(seq_ids), num_seqs, window, hq, float(scale), int(agg),
                               _ptr(scores), _ptr(ws), ws.numel(), _ptr(status),
                               _stream(stream)), "kara_score_ex")
    return scores


def kara_select_chunks(scores: torch.Tensor, k: int, anchor_frac: float, gap_limit: int,
                       widen: int, keep: torch.Tensor | None = None,
                       sel: torch.Tensor | None = None, trim: int = TRIM_TOKEN,
                       stream=None) -> torch.Tensor:
    """kara_select + kara_token2chunk in one kernel: keep [..., k] int32 (sel, if given, gets
    the selection). trim=TRIM_CHUNK runs kara_select_chunks_ex with the chunk-aware trim."""
    _require(scores, torch.float32, "scores")
    w = scores.shape[-1]
    rows = scores.numel() // w if w else 0
    if keep is None:
        keep = torch.empty(scores.shape[:-1] + (k,), dtype=torch.int32, device=scores.device)
    _require(keep, torch.int32, "keep")
    if sel is not None:
        _require(sel, torch.int32, "sel")
    if trim == TRIM_TOKEN:
        _check(lib().kara_select_chunks(_ptr(scores), rows, w, k, float(anchor_frac), gap_limit,
                                        widen, _ptr(sel), _ptr(keep), _stream(stream)),
               "kara_select_chunks")
    else:
        _check(lib().kara_select_chunks_ex(_ptr(scores), rows, w, k, float(anchor_frac),
                                           gap_limit, widen, int(trim), _ptr(sel), _ptr(keep),
                                           _stream(stream)), "kara_select_chunks_ex")
    return keep


def kara_compress(scores: torch.Tensor, k_layers, v_layers, pool: PagedPool, window: int, k: int,
                  anchor_frac: float, gap_limit: int, widen: int,
                  seq_ids: torch.Tensor | None = None, keep: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                  stream=None) -> torch.Tensor:
    """Selection, Token2Chunk and compaction of all layers from their scores
    [L, R, Hkv, W] (in place on the pools and the PagedPool). Returns the status tensor."""
    _require(scores, torch.float32, "scores")
    nl, r, hkv, w = scores.shape
    arr = _layers(k_layers, v_layers)
    if nl != len(arr) or w != window:
        raise ValueError("scores must be [layers, sequences, KV heads, window]")
    if seq_ids is not None:
        _require(seq_ids, torch.int32, "seq_ids")
    if keep is not None:
        _require(keep, torch.int32, "keep")
    status = _status(status, scores.device)
    ps = pool.c_struct()
    ws = _workspace(kara_workspace_bytes(OP_COMPACT, pool, r, window, 0, k), scores.device,
                    workspace)
    _check(lib().kara_compress(_ptr(scores), arr, nl, ctypes.byref(ps), _ptr(seq_ids), r, window,
                               k, float(anchor_frac), gap_limit, widen, _ptr(keep), _ptr(ws),
                               ws.numel(), _ptr(status), _stream(stream)), "kara_compress")
    return status


def kara_sum_heads(scores: torch.Tensor, out: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """[..., Hkv, W] scores summed over the heads: [..., W] fp32."""
    _require(scores, torch.float32, "scores")
    hkv, w = scores.shape[-2], scores.shape[-1]
    rows = scores.numel() // (hkv * w) if hkv * w else 0
    if out is None:
        out = torch.empty(scores.shape[:-2] + (w,), dtype=torch.float32, device=scores.device)
    _require(out, torch.float32, "out")
    _check(lib().kara_sum_heads(_ptr(scores), rows, hkv, w, _ptr(out), _stream(stream)),
           "kara_sum_heads")
    return out


def kara_expand_keep(keep_shared: torch.Tensor, num_kv_heads: int,
                     keep: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """[..., k] keep sets copied to every KV head: [..., Hkv, k] int32."""
    _require(keep_shared, torch.int32, "keep_shared")
    k = keep_shared.shape[-1]
    rows = keep_shared.numel() // k if k else 0
    if keep is None:
        keep = torch.empty(keep_shared.shape[:-1] + (num_kv_heads, k), dtype=torch.int32,
                           device=keep_shared.device)
    _require(keep, torch.int32, "keep")
    _check(lib().kara_expand_keep(_ptr(keep_shared), rows, num_kv_heads, k, _ptr(keep),
                                  _stream(stream)), "kara_expand_keep")
    return keep


def kara_select(scores: torch.Tensor, k: int, sel: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """Top-k window positions per row, ascending: [..., k] int32."""
    _require(scores, torch.float32, "scores")
    w = scores.shape[-1]
    rows = scores.numel() // w if w else 0
    if sel is None:
        sel = torch.empty(scores.shape[:-1] + (k,), dtype=torch.int32, device=scores.device)
    _require(sel, torch.int32, "sel")
    _check(lib().kara_select(_ptr(scores), rows, w, k, _ptr(sel), _stream(stream)), "kara_select")
    return sel


def kara_token2chunk(scores: torch.Tensor, sel: torch.Tensor, anchor_frac: float, gap_limit: int,
                     widen: int, keep: torch.Tensor | None = None, trim: int = TRIM_TOKEN,
                     stream=None) -> torch.Tensor:
    """Token2Chunk expansion and trim with ceil(anchor_frac * k) anchors: [..., k] int32
    ascending. trim=TRIM_CHUNK runs kara_token2chunk_ex with the chunk-aware trim."""
    _require(scores, torch.float32, "scores")
    _require(sel, torch.int32, "sel")
    w = scores.shape[-1]
    k = sel.shape[-1]
    rows = scores.numel() // w if w else 0
    if keep is None:
        keep = torch.empty_like(sel)
    _require(keep, torch.int32, "keep")
    if trim == TRIM_TOKEN:
        _check(lib().kara_token2chunk(_ptr(scores), _ptr(sel), rows, w, k, float(anchor_frac),
                                      int(gap_limit), int(widen), _ptr(keep), _stream(stream)),
               "kara_token2chunk")
    else:
        _check(lib().kara_token2chunk_ex(_ptr(scores), _ptr(sel), rows, w, k, float(anchor_frac),
                                         int(gap_limit), int(widen), int(trim), _ptr(keep),
                                         _stream(stream)), "kara_token2chunk_ex")
    return keep


def _layers(k_layers, v_layers):
    if len(k_layers) != len(v_layers) or not 1 <= len(k_layers) <= MAX_LAYERS:
        raise ValueError("k_layers and v_layers must hold 1..128 tensors each")
    arr = (_LayerKV * len(k_layers))()
    for i, (k, v) in enumerate(zip(k_layers, v_layers)):
        _require(k, torch.bfloat16, f"k_layers[{i}]")
        _require(v, torch.bfloat16, f"v_layers[{i}]")
        arr[i].k = k.data_ptr()
        arr[i].v = v.data_ptr()
    return arr


def kara_compact(k_layers, v_layers, pool: PagedPool, window: int, keep: torch.Tensor,
                 seq_ids: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                 status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Compaction into fresh blocks (in place on the pools and the PagedPool). Returns the
    status tensor (read it after synchronising)."""
    _require(keep, torch.int32, "keep")
    nl, r, hkv, k = keep.shape
    arr = _layers(k_layers, v_layers)
    if nl != len(arr):
        raise ValueError("keep's first dimension must equal the number of layers")
    if seq_ids is not None:
        _require(seq_ids, torch.int32, "seq_ids")
    status = _status(status, keep.device)
    ps = pool.c_struct()
    nbytes = kara_workspace_bytes(OP_COMPACT, pool, r, window, 0, k)
    ws = _workspace(nbytes, keep.device, workspace)
    _check(lib().kara_compact(arr, nl, ctypes.byref(ps), _ptr(seq_ids), r, window, k, _ptr(keep),
                              _ptr(ws), ws.numel(), _ptr(status), _stream(stream)),
           "kara_compact")
    return status


def kara_compact_noalloc(k_layers, v_layers, pool: PagedPool, window: int, keep: torch.Tensor,
                         seq_ids: torch.Tensor | None = None, status: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """kara_compact with the plan scratch in the library's fixed device array: the call
    allocates no device memory (for callers that cannot allocate when they compress). Returns
    the status tensor; raises KaraError(ERR_WORKSPACE) when the plan would not fit."""
    _require(keep, torch.int32, "keep")
    nl, r, hkv, k = keep.shape
    arr = _layers(k_layers, v_layers)
    if nl != len(arr):
        raise ValueError("keep's first dimension must equal the number of layers")
    if seq_ids is not None:
        _require(seq_ids, torch.int32, "seq_ids")
    if status is None:
        raise ValueError("pass a preallocated status tensor (this call allocates nothing)")
    _require(status, torch.int32, "status")
    ps = pool.c_struct()
    _check(lib().kara_compact_noalloc(arr, nl, ctypes.byref(ps), _ptr(seq_ids), r, window, k,
                                      _ptr(keep), _ptr(status), _stream(stream)),
           "kara_compact_noalloc")
    return status


def paged_decode_attn(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                      pool: PagedPool, scale: float | None = None, out: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """One decode step of paged GQA attention: out [B, Hq, d] bf16."""
    _require(q, torch.bfloat16, "q")
    _require(k_cache, torch.bfloat16, "k_cache")
    _require(v_cache, torch.bfloat16, "v_cache")
    b, hq, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    _require(out, torch.bfloat16, "out")
    status = _status(status, q.device)
    ps = pool.c_struct()
    nbytes = kara_workspace_bytes(OP_DECODE, pool, 0, 0, hq, 0)
    ws = _workspace(nbytes, q.device, workspace)
    _check(lib().paged_decode_attn(_ptr(q), _ptr(k_cache), _ptr(v_cache), ctypes.byref(ps), hq,
                                   float(scale), _ptr(out), _ptr(ws), ws.numel(), _ptr(status),
                                   _stream(stream)), "paged_decode_attn")
    return out


def kara_score_ring(q_ring: torch.Tensor, k_cache: torch.Tensor, pool: PagedPool, window: int,
                    seq_ids: torch.Tensor, num_seqs: int, scale: float | None = None,
                    scores: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                    status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Window scores [num_seqs, Hkv, W] fp32 with the queries read from the window-query ring
    q_ring [B, 2W, Hq, d] (see kara_score_ring in include/kara.h)."""
    _require(q_ring, torch.bfloat16, "q_ring")
    _require(k_cache, torch.bfloat16, "k_cache")
    _require(seq_ids, torch.int32, "seq_ids")
    b, rows, hq, d = q_ring.shape
    if rows != 2 * window:
        raise ValueError("q_ring's second dimension must be 2 * window")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if scores is None:
        scores = torch.empty((num_seqs, pool.num_kv_heads, window), dtype=torch.float32,
                             device=q_ring.device)
    _require(scores, torch.float32, "scores")
    status = _status(status, q_ring.device)
    ps = pool.c_struct()
    ws = _workspace(kara_workspace_bytes(OP_SCORE, pool, num_seqs, window, hq), q_ring.device,
                    workspace)
    _check(lib().kara_score_ring(_ptr(q_ring), _ptr(k_cache), ctypes.byref(ps), _ptr(seq_ids),
                                 num_seqs, window, hq, float(scale), _ptr(scores), _ptr(ws),
                                 ws.numel(), _ptr(status), _stream(stream)), "kara_score_ring")
    return scores


def kara_decode_append(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                       k_cache: torch.Tensor, v_cache: torch.Tensor, pool: PagedPool,
                       q_ring: torch.Tensor | None = None, window: int = 0,
                       scale: float | None = None, out: torch.Tensor | None = None,
                       workspace: torch.Tensor | None = None, status: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """One layer of a decode step, fused: attention of the new token (slot ctx_len) over the
    cache and itself, its K/V written to the cache and its query to the ring. out [B, Hq, d]."""
    for t, name in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_cache, "k_cache"),
                    (v_cache, "v_cache")):
        _require(t, torch.bfloat16, name)
    if q_ring is not None:
        _require(q_ring, torch.bfloat16, "q_ring")
    b, hq, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    _require(out, torch.bfloat16, "out")
    status = _status(status, q.device)
    ps = pool.c_struct()
    ws = _workspace(kara_workspace_bytes(OP_DECODE, pool, 0, 0, hq, 0), q.device, workspace)
    _check(lib().kara_decode_append(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                    _ptr(v_cache), ctypes.byref(ps), hq, float(scale),
                                    _ptr(q_ring), int(window), _ptr(out), _ptr(ws), ws.numel(),
                                    _ptr(status), _stream(stream)), "kara_decode_append")
    return out


def kara_step_begin(pool: PagedPool, status: torch.Tensor, stream=None) -> None:
    """Blocks for the slots a decode step appends (see include/kara.h)."""
    _require(status, torch.int32, "status")
    ps = pool.c_struct()
    _check(lib().kara_step_begin(ctypes.byref(ps), _ptr(status), _stream(stream)),
           "kara_step_begin")


def kara_step_end(pool: PagedPool, tail: torch.Tensor | None = None, window: int = 0,
                  check: bool = False, due: torch.Tensor | None = None,
                  due_count: torch.Tensor | None = None, capacity: int = 0,
                  stream=None) -> None:
    """ctx_len + 1 and tail + 1; on a check step the due sequences (tail >= window, or
    ctx_len >= capacity) and their count."""
    if tail is not None:
        _require(tail, torch.int32, "tail")
    for t, name in ((due, "due"), (due_count, "due_count")):
        if t is not None:
            _require(t, torch.int32, name)
    ps = pool.c_struct()
    _check(lib().kara_step_end(ctypes.byref(ps), _ptr(tail), int(window), int(capacity),
                               1 if check else 0, _ptr(due), _ptr(due_count), _stream(stream)),
           "kara_step_end")


def kara_reset_tails(tail: torch.Tensor, seq_ids: torch.Tensor, num_seqs: int,
                     stream=None) -> None:
    _require(tail, torch.int32, "tail")
    _require(seq_ids, torch.int32, "seq_ids")
    _check(lib().kara_reset_tails(_ptr(tail), _ptr(seq_ids), int(num_seqs), int(tail.numel()),
                                  _stream(stream)), "kara_reset_tails")


def lacache_compact(k_layers, v_layers, pool: PagedPool, span: int, overlap: int, rung: int,
                    budget: int, sink: int = 0, recent: int = 0,
                    seq_ids: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                    status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One ladder-compaction pass (in place). Returns the status tensor."""
    arr = _layers(k_layers, v_layers)
    device = k_layers[0].device
    r = int(seq_ids.numel()) if seq_ids is not None else int(pool.block_table.shape[0])
    if seq_ids is not None:
        _require(seq_ids, torch.int32, "seq_ids")
    status = _status(status, device)
    ps = pool.c_struct()
    prm = _LacacheParams(span, overlap, rung, budget, sink, recent)
    nbytes = kara_workspace_bytes(OP_LACACHE, pool, r, 0, 0, budget)
    ws = _workspace(nbytes, device, workspace)
    _check(lib().lacache_compact(arr, len(arr), ctypes.byref(ps), _ptr(seq_ids), r,
                                 ctypes.byref(prm), _ptr(ws), ws.numel(), _ptr(status),
                                 _stream(stream)), "lacache_compact")
    return status


def kara_wait_probe(wait_ms: int, status: torch.Tensor | None = None, device="cuda",
                    stream=None) -> torch.Tensor:
    """Runs the bounded-wait probe (a wait that times out after about `wait_ms`). Returns the
    status tensor, which holds KARA_ERR_TIMEOUT once the stream completes."""
    status = _status(status, torch.device(device))
    _check(lib().kara_wait_probe(int(wait_ms), _ptr(status), _stream(stream)), "kara_wait_probe")
    return status

