"""The C-ABI library: it builds, loads without a GPU, exports every declared entry point, and
rejects bad arguments on the host before touching the device (no compute calls here)."""

import ctypes

import pytest

from decode_kv_cache_kara_b200 import kara as K


def test_library_exports_every_declared_symbol(lib_path):
    names = K.declared_symbols()
    expected = {"kara_score", "kara_select", "kara_token2chunk", "kara_compact",
                "paged_decode_attn", "lacache_compact", "kara_workspace_bytes",
                "kara_status_str", "kara_version", "kara_launch_count"}
    assert expected <= set(names)
    handle = ctypes.CDLL(lib_path)
    for n in names:
        assert hasattr(handle, n), n


def test_status_strings_and_version(lib_path):
    assert K.status_str(0) == "ok"
    assert "free blocks" in K.status_str(K.ERR_OUT_OF_BLOCKS)
    assert K.lib().kara_version().decode().startswith("kara-b200")


def test_host_side_validation_returns_before_any_launch(lib_path):
    L = K.lib()
    launches = K.kara_launch_count()
    null = ctypes.c_void_p(0)
    # k > window, window too large, rows < 0
    assert L.kara_select(null, 4, 16, 17, null, null) == K.ERR_INVALID_ARG
    assert L.kara_select(null, 4, 5000, 8, null, null) == K.ERR_INVALID_ARG
    assert L.kara_select(null, 0, 16, 4, null, null) == K.OK          # empty input
    # an unknown trim
    assert L.kara_token2chunk_ex(null, null, 1, 16, 4, 0.5, 8, 1, 2, null, null) == K.ERR_INVALID_ARG
    assert L.kara_select_chunks_ex(null, 1, 16, 4, 0.5, 8, 1, -1, null, null, null) == K.ERR_INVALID_ARG
    assert L.kara_select_chunks_ex(null, 0, 16, 4, 0.5, 8, 1, K.TRIM_CHUNK, null, null, null) == K.OK
    # anchor fractions outside [0, 1] (and NaN)
    for frac in (5.0, 1.01, -0.1, float("nan")):
        assert L.kara_token2chunk(null, null, 1, 16, 4, frac, 8, 1, null, null) == K.ERR_INVALID_ARG
    # page size other than 16, head_dim other than 64/128
    pool = K._Pool(1, 1, 1, 1, 1, 8, 64, 8, 2, 128)
    assert L.paged_decode_attn(null, null, null, ctypes.byref(pool), 4, 1.0, null, null, 0, null,
                               null) == K.ERR_UNSUPPORTED
    pool = K._Pool(1, 1, 1, 1, 1, 8, 64, 16, 2, 96)
    assert L.kara_score(null, null, ctypes.byref(pool), null, 1, 16, 4, 1.0, null, null, 0, null,
                        null) == K.ERR_UNSUPPORTED
    # more than 8 query heads per KV head
    pool = K._Pool(1, 1, 1, 1, 1, 8, 64, 16, 2, 128)
    assert L.kara_score(null, null, ctypes.byref(pool), null, 1, 16, 18, 1.0, null, null, 0, null,
                        null) == K.ERR_UNSUPPORTED
    # workspace missing
    one = ctypes.c_void_p(256)
    assert L.kara_score(one, one, ctypes.byref(pool), null, 1, 16, 4, 1.0, one, null, 0, one,
                        null) == K.ERR_WORKSPACE
    # LaCache: stride S-O must divide S and L
    prm = K._LacacheParams(3, 1, 4, 64, 0, 0)
    layers = (K._LayerKV * 8)()
    assert L.lacache_compact(layers, 8, ctypes.byref(pool), null, 1, ctypes.byref(prm), null, 0,
                             one, null) == K.ERR_INVALID_ARG
    # the wait probe: budget outside 1..2000 ms, or no status buffer
    assert L.kara_wait_probe(0, one, null) == K.ERR_INVALID_ARG
    assert L.kara_wait_probe(2001, one, null) == K.ERR_INVALID_ARG
    assert L.kara_wait_probe(100, null, null) == K.ERR_INVALID_ARG
    # compaction window above KARA_MAX_WINDOW
    assert L.kara_compact(layers, 1, ctypes.byref(pool), null, 1, 5000, 8, one, one, 1 << 20, one,
                          null) == K.ERR_INVALID_ARG
    # decode loop: a check step needs the tail and due buffers; the fused step needs the new
    # token; a ring needs a window in range; negative counts
    assert L.kara_step_end(ctypes.byref(pool), null, 16, 0, 1, one, one, null) == K.ERR_INVALID_ARG
    assert L.kara_step_end(ctypes.byref(pool), null, 0, 0, 1, one, one, null) == K.ERR_INVALID_ARG
    assert L.kara_decode_append(one, null, one, one, one, ctypes.byref(pool), 4, 1.0, null, 0, one,
                                one, 1 << 20, one, null) == K.ERR_INVALID_ARG
    assert L.kara_decode_append(one, one, one, one, one, ctypes.byref(pool), 4, 1.0, one, 0, one,
                                one, 1 << 20, one, null) == K.ERR_INVALID_ARG
    assert L.kara_reset_tails(one, one, -1, 4, null) == K.ERR_INVALID_ARG
    assert L.kara_reset_tails(one, one, 0, 4, null) == K.OK             # nothing to reset
    assert L.kara_score_ring(one, one, ctypes.byref(pool), null, 1, 5000, 4, 1.0, one, one,
                             1 << 20, one, null) == K.ERR_INVALID_ARG
    # fused selection: an anchor fraction above 1, k above the window; fused compression: the
    # same, and a missing free list
    assert L.kara_select_chunks(one, 2, 64, 8, 9.0, 8, 1, null, one, null) == K.ERR_INVALID_ARG
    assert L.kara_select_chunks(one, 2, 64, 65, 0.5, 8, 1, null, one, null) == K.ERR_INVALID_ARG
    assert L.kara_select_chunks(one, 0, 64, 8, 0.5, 8, 1, null, one, null) == K.OK
    assert L.kara_compress(one, layers, 1, ctypes.byref(pool), null, 1, 64, 8, 1.5, 8, 1, null,
                           one, 1 << 20, one, null) == K.ERR_INVALID_ARG
    nofree = K._Pool(1, 1, 0, 0, 1, 8, 64, 16, 2, 128)
    assert L.kara_compress(one, layers, 1, ctypes.byref(nofree), null, 1, 64, 8, 0.5, 8, 1, null,
                           one, 1 << 20, one, null) == K.ERR_INVALID_ARG
    # none of these reached a kernel launch
    assert K.kara_launch_count() == launches


def test_workspace_sizes(lib_path):
    pool = K._Pool(1, 1, 1, 1, 32, 257, 9000, 16, 4, 128)
    score = K.lib().kara_workspace_bytes(K.OP_SCORE, None, 32, 1000, 28, 0)
    assert score == 32 * 28 * 5 * 1024 * 4            # 4 key chunks + merged, rows padded to 256
    assert K.lib().kara_workspace_bytes(K.OP_SCORE, None, 1, 1024, 1, 0) == 6 * 1024 * 4
    dec = K.lib().kara_workspace_bytes(K.OP_DECODE, ctypes.byref(pool), 0, 0, 28, 0)
    assert dec == 32 * 28 * 33 * 130 * 4              # 33 units of 8 pages, d + 2 floats
    comp = K.lib().kara_workspace_bytes(K.OP_COMPACT, None, 32, 1024, 0, 204)
    assert comp == (144 + 32 * 12 + 32 * 14) * 4      # header with the keep check's verdicts


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(K, "_LIB", None)
    monkeypatch.setattr(K, "library_path", lambda: str(tmp_path / "nope.so"))
    with pytest.raises(K.KaraLibraryError):
        K.lib()


def test_binding_refuses_host_tensors():
    """No CPU fallback: every compute call of the binding refuses host tensors before it
    reaches the library (there is no other path to take)."""
    import torch

    w, k = 32, 8
    s = torch.zeros((2, 2, w))
    q = torch.zeros((2, w, 4, 64), dtype=torch.bfloat16)
    kv = torch.zeros((4, 16, 2, 64), dtype=torch.bfloat16)
    sel = torch.zeros((2, 2, k), dtype=torch.int32)
    ring = torch.zeros((2, 2 * w, 4, 64), dtype=torch.bfloat16)
    seq = torch.zeros(2, dtype=torch.int32)
    status = torch.zeros(1, dtype=torch.int32)
    pool = K.PagedPool(torch.zeros((2, 4), dtype=torch.int32), torch.zeros(2, dtype=torch.int32),
                       torch.zeros(4, dtype=torch.int32), torch.zeros(1, dtype=torch.int32), 4, 2,
                       64)
    calls = {
        "kara_score": lambda: K.kara_score(q, kv, pool, w),
        "kara_score_ex": lambda: K.kara_score_ex(q, kv, pool, w),
        "kara_select": lambda: K.kara_select(s, k),
        "kara_token2chunk": lambda: K.kara_token2chunk(s, sel, 0.5, 8, 1),
        "kara_select_chunks": lambda: K.kara_select_chunks(s, k, 0.5, 8, 1),
        "kara_sum_heads": lambda: K.kara_sum_heads(s),
        "kara_expand_keep": lambda: K.kara_expand_keep(sel[:, 0].contiguous(), 2),
        "kara_compact": lambda: K.kara_compact([kv], [kv], pool, w, sel[None]),
        "kara_compress": lambda: K.kara_compress(s[None], [kv], [kv], pool, w, k, 0.5, 8, 1),
        "kara_compact_noalloc": lambda: K.kara_compact_noalloc([kv], [kv], pool, w, sel[None],
                                                               status=status),
        "lacache_compact": lambda: K.lacache_compact([kv], [kv], pool, 1, 0, 16, 64),
        "paged_decode_attn": lambda: K.paged_decode_attn(q[:, 0], kv, kv, pool),
        "kara_decode_append": lambda: K.kara_decode_append(q[:, 0], kv[0], kv[0], kv, kv, pool),
        "kara_score_ring": lambda: K.kara_score_ring(ring, kv, pool, w, seq, 2),
        "kara_step_begin": lambda: K.kara_step_begin(pool, status),
        "kara_step_end": lambda: K.kara_step_end(pool, seq, w, True, seq, seq[:1]),
        "kara_reset_tails": lambda: K.kara_reset_tails(seq, seq, 2),
        # a host status word or workspace is refused as well (its address is no device address)
        "kara_wait_probe": lambda: K.kara_wait_probe(100, status=status),
    }
    for name, fn in calls.items():
        with pytest.raises(ValueError, match="CUDA tensor"):
            fn()


def test_empty_inputs_return_ok_without_a_launch(lib_path):
    """No rows, no due sequences, an empty batch: every compute call returns KARA_OK on the
    host and launches nothing (the buffers are never touched, so null pointers do)."""
    L = K.lib()
    null = ctypes.c_void_p(0)
    launches = K.kara_launch_count()
    pool = K._Pool(8, 8, 8, 8, 3, 64, 64, 16, 2, 128)       # dummy table pointers, 3 sequences
    empty = K._Pool(8, 8, 8, 8, 0, 64, 64, 16, 2, 128)      # no sequence at all
    layers = (K._LayerKV * 1)()
    prm = K._LacacheParams(2, 1, 64, 2048, 64, 64)
    calls = {
        "kara_score": L.kara_score(null, null, ctypes.byref(pool), null, 0, 16, 4, 1.0, null,
                                   null, 0, null, null),
        "kara_score_ex max": L.kara_score_ex(null, 0, null, ctypes.byref(pool), null, 0, 16, 4,
                                             1.0, K.AGG_MAX, null, null, 0, null, null),
        "kara_score_ring": L.kara_score_ring(null, null, ctypes.byref(pool), null, 0, 16, 4, 1.0,
                                             null, null, 0, null, null),
        "kara_token2chunk": L.kara_token2chunk(null, null, 0, 16, 4, 0.5, 8, 1, null, null),
        "kara_select_chunks": L.kara_select_chunks(null, 0, 16, 4, 0.5, 8, 1, null, null, null),
        "kara_sum_heads": L.kara_sum_heads(null, 0, 2, 16, null, null),
        "kara_expand_keep": L.kara_expand_keep(null, 0, 2, 4, null, null),
        "kara_compact": L.kara_compact(layers, 1, ctypes.byref(pool), null, 0, 16, 4, null, null,
                                       0, null, null),
        "kara_compress": L.kara_compress(null, layers, 1, ctypes.byref(pool), null, 0, 16, 4, 0.5,
                                         8, 1, null, null, 0, null, null),
        "lacache_compact": L.lacache_compact(layers, 4, ctypes.byref(pool), null, 0,
                                             ctypes.byref(prm), null, 0, null, null),
        "paged_decode_attn": L.paged_decode_attn(null, null, null, ctypes.byref(empty), 4, 1.0,
                                                 null, null, 0, null, null),
    }
    assert {name: code for name, code in calls.items() if code != K.OK} == {}
    assert K.kara_launch_count() == launches
