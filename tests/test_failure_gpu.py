"""Failure detection on the GPU without a fault: a bounded wait that runs out.

kara_wait_probe runs the library's bounded mbarrier wait on barriers that nothing arrives on:
one waiter with a short budget times out, reports KARA_ERR_TIMEOUT and raises the CTA's abort
flag; a second waiter with the default budget (about 2 s) must leave through that flag. The
host reads the status, and the context stays usable for the next call.
"""
import time

import numpy as np
import pytest
import torch

from decode_kv_cache_kara_b200 import kara as K
from oracle import kara as ok

pytestmark = pytest.mark.gpu


def test_wait_probe_times_out_and_context_stays_usable():
    dev = torch.device("cuda")
    torch.cuda.synchronize()
    status = K.new_status(dev)
    t0 = time.perf_counter()
    K.kara_wait_probe(100, status=status, device=dev)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert K.read_status(status) == K.ERR_TIMEOUT
    # the second waiter left through the abort flag, well before its own 2 s budget
    assert dt < 1.5, dt
    # the context is still usable: a selection right after matches the oracle
    g = torch.Generator(device="cpu").manual_seed(7)
    scores = torch.rand((6, 96), generator=g, dtype=torch.float32)
    sel = K.kara_select(scores.to(dev), 12)
    torch.cuda.synchronize()
    got = sel.cpu().numpy()
    for r in range(scores.shape[0]):
        assert np.array_equal(got[r], ok.select_topk(scores[r].double().numpy(), 12))


def test_wait_probe_status_is_sticky_first_error():
    dev = torch.device("cuda")
    status = K.new_status(dev)
    status.fill_(K.ERR_BAD_BLOCK)           # an earlier error stays the reported one
    K.kara_wait_probe(10, status=status, device=dev)
    torch.cuda.synchronize()
    assert K.read_status(status) == K.ERR_BAD_BLOCK
