"""Failure detection on the GPU without a fault: a bounded wait that nothing satisfies gives up,
records ISKV_ERR_TIMEOUT in the history's status word, and leaves the context usable."""

import time

import numpy as np
import pytest
import torch

from gpu_util import bit, kv, state, stored
import synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    m = kv()
    h = m.LowRankHistory(128, 16, 64, storage=torch.float32)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    m.selftest_wait_timeout(h, 20_000_000)  # 20 ms
    k, n, folds, st = h.status()
    elapsed = time.perf_counter() - t0
    assert st == bit(7)                      # ISKV_ERR_TIMEOUT, nothing else
    assert 0.02 <= elapsed < 5.0
    # The context still runs work: a fold on another history succeeds.
    g = m.LowRankHistory(128, 16, 64, storage=torch.float32)
    X = stored(synth.lowrank_rows(32, 128, 1.0, 0.01, seed=0), torch.float32)
    Xd = torch.as_tensor(X, dtype=torch.float32, device="cuda")
    m.fold_block(g, Xd[:16].contiguous(), torch.arange(16, dtype=torch.int32, device="cuda"))
    assert g.status()[3] == 0 and g.status()[1] == 16
