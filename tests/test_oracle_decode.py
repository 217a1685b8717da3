"""Pins of the paged decode-attention oracle."""

import math

import numpy as np
import pytest
import torch

from oracle import decode as od


def paged(seed, page=4, nb=10, hkv=2, d=8):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((nb, page, hkv, d)), rng.standard_normal((nb, page, hkv, d))


def test_single_slot_returns_its_value_row():
    kp, vp = paged(0)
    q = np.random.default_rng(1).standard_normal((1, 4, 8))
    out = od.decode_attention(q, kp, vp, np.array([[6, 1]]), np.array([1]), 0.3, 4)
    for h in range(4):
        assert np.allclose(out[0, h], vp[6, 0, h // 2], rtol=0, atol=1e-15)


def test_equal_scores_average_the_values():
    kp, vp = paged(2)
    kp[:] = 0.0
    q = np.random.default_rng(3).standard_normal((1, 2, 8))
    table = np.array([[3, 7, 1]])
    out = od.decode_attention(q, kp, vp, table, np.array([10]), 1.0, 4)
    slots = np.arange(10)
    v = vp[table[0][slots // 4], slots % 4]
    assert np.allclose(out[0, 0], v[:, 0].mean(axis=0), atol=1e-14)
    assert np.allclose(out[0, 1], v[:, 1].mean(axis=0), atol=1e-14)


def test_empty_context_is_zero():
    kp, vp = paged(4)
    out = od.decode_attention(np.ones((1, 2, 8)), kp, vp, np.array([[0]]), np.array([0]), 1.0, 4)
    assert (out == 0).all()


@pytest.mark.parametrize("seed", range(4))
def test_matches_torch_sdpa_on_contiguous_copy(seed):
    rng = np.random.default_rng(10 + seed)
    page, hkv, hq, d = 4, 2, 6, 8
    ctx = rng.integers(1, 30, size=3)
    pages = [-(-int(n) // page) for n in ctx]
    nb = sum(pages) + 3
    perm = rng.permutation(nb)
    table = np.full((3, max(pages)), -1)
    pos = 0
    for b in range(3):
        table[b, :pages[b]] = perm[pos:pos + pages[b]]
        pos += pages[b]
    kp, vp = paged(seed, page, nb, hkv, d)
    q = rng.standard_normal((3, hq, d))
    scale = 1 / math.sqrt(d)
    out = od.decode_attention(q, kp, vp, table, ctx, scale, page)
    for b in range(3):
        n = int(ctx[b])
        s = np.arange(n)
        k = torch.from_numpy(kp[table[b][s // page], s % page]).permute(1, 0, 2)   # [Hkv, n, d]
        v = torch.from_numpy(vp[table[b][s // page], s % page]).permute(1, 0, 2)
        k = k.repeat_interleave(hq // hkv, 0)
        v = v.repeat_interleave(hq // hkv, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b])[:, None, :], k, v, scale=scale)[:, 0, :]
        assert np.allclose(out[b], ref.numpy(), rtol=1e-12, atol=1e-13)


def test_block_placement_does_not_matter():
    # Moving the blocks of a sequence to other ids (and the table with them) changes nothing.
    kp, vp = paged(5, nb=8)
    q = np.random.default_rng(6).standard_normal((1, 4, 8))
    t1 = np.array([[2, 5, 7]])
    perm = np.array([4, 0, 6, 1, 3, 2, 7, 5])                  # new id of old block i
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    t2 = perm[t1]
    a = od.decode_attention(q, kp, vp, t1, np.array([11]), 0.5, 4)
    b = od.decode_attention(q, kp2, vp2, t2, np.array([11]), 0.5, 4)
    assert np.array_equal(a, b)
