"""Failure reporting of the kernels' bounded waits, on the GPU, without a fault.

Every mbarrier wait in the library gives up after a time limit, records code 1 in the workspace status
word and lets its kernel finish.  The self-test entry point runs that wait routine on a barrier nothing
completes, with a short limit; the host must read the code, and the context must stay usable.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_indexer_04_b200 as dsa
import workloads
from gpu_util import Dev

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda:0")
    dsa.selftest_wait_timeout(2000, ws)            # 2 ms
    assert dsa.device_check(ws) == 1               # "a wait ran out", read by the host
    assert dsa.device_check(ws) == 0               # the check cleared it
    # the context is still usable: an exact computation afterwards is right
    b = workloads.tiny_integer(seed=0, T=256, H=4, d=32, k=32)
    idx = Dev(b).topk(32)
    ref = oracle.dense(b, k=32)
    for t in range(b.n_q):
        assert set(idx[t][idx[t] >= 0].tolist()) == set(ref["idx"][t][ref["idx"][t] >= 0].tolist())


def test_selftest_rejects_bad_arguments():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda:0")
    for limit in (0, 2_000_000):
        with pytest.raises(dsa.DsaError):
            dsa.selftest_wait_timeout(limit, ws)
