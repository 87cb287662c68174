"""Failure detection without a GPU fault: the bounded wait every on-chip
pipeline uses gives up on a barrier that never completes, records
MISA_DEV_WAIT_TIMEOUT in the status word and returns; the context stays
usable and a normal call afterwards is correct."""
import time

import numpy as np
import pytest
import torch

from long_context_misa_b200 import inputs as G
from long_context_misa_b200 import misa as M
from tests.parity import to_device

pytestmark = pytest.mark.gpu


def test_bounded_wait_records_timeout_and_returns():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    M.debug_wait_timeout(status, 20_000_000)  # 20 ms
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert int(status.item()) & M.DEV_WAIT_TIMEOUT
    assert elapsed < 5.0
    # the context is intact: an ordinary call still works and is correct
    wl = G.WORKLOADS["tiny_decode"].scaled(L=1000, k=50)
    inp = G.make_inputs(wl, 0)
    cache, qs = to_device(inp, torch)
    a = M.dense_score_topk(cache, qs, wl.k).cpu().numpy()
    b = M.dense_score_topk(cache, qs, wl.k).cpu().numpy()
    assert np.array_equal(a, b) and (a >= 0).sum() == wl.k
    assert cache.device_status() == 0
