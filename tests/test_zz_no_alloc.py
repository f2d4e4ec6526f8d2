"""The allocation-free dense top-k (dsa_index_topk_static) against the
workspace entry point (dsa_index_topk).

It exists for callers that cannot allocate device memory, e.g. a custom-op
callback of an inference runtime that gets no allocator.  Its workspace is a
device array inside the library shared by every call, so the test makes two
calls in a row (the second sees the first call's leftovers) and compares each
with dsa_index_topk on the same inputs.  This file sorts last so that a run
stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_indexer_04_b200 as dsa
import workloads

pytestmark = pytest.mark.gpu


def call_static(lay, Q, K, W, k):
    """Through the C ABI directly."""
    idx = torch.full((lay.num_queries, k), -7, dtype=torch.int32, device=lay.device)
    sc = torch.full((lay.num_queries, k), 7.0, dtype=torch.float32, device=lay.device)
    st = dsa.library().dsa_index_topk_static(lay.ref(), ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
                                             ctypes.c_void_p(W.data_ptr()), k, ctypes.c_void_p(idx.data_ptr()),
                                             ctypes.c_void_p(sc.data_ptr()),
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, dsa.library().dsa_status_string(st)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("make,k", [
    (lambda: workloads.tiny_integer(seed=0, T=512, H=4, d=32, k=64), 64),        # exact integer scores
    (lambda: workloads.dense_decode(seed=5, B=4, L=6000, n_mtp=2, H=64, d=128, k=512), 512),
])
def test_static_scratch_matches_workspace_entry_point(make, k):
    b = make()
    dev = torch.device("cuda:0")
    lay = dsa.Layout.from_batch(b, dev)
    Q, K, W = b.Q.to(dev), b.K.to(dev), b.W.to(dev)
    ref_idx, ref_sc = dsa.index_topk(lay, Q, K, W, k, want_scores=True)
    torch.cuda.synchronize()
    ref_idx, ref_sc = ref_idx.cpu().numpy(), ref_sc.cpu().numpy()
    for call in range(2):
        idx, sc = call_static(lay, Q, K, W, k)
        assert np.array_equal(idx, ref_idx), f"call {call}: indices differ"
        assert np.array_equal(np.isnan(sc), np.isnan(ref_sc))
        v = ~np.isnan(ref_sc)
        assert np.array_equal(sc[v], ref_sc[v]), f"call {call}: scores differ"


def test_static_scratch_rejects_batches_beyond_capacity():
    cap = dsa.index_topk_static_capacity()
    b = workloads.dense_decode(seed=6, B=8, L=40000, n_mtp=8, H=64, d=128, k=64)   # 64 rows x 40000 scores
    lay = dsa.Layout.from_batch(b, torch.device("cuda:0"))
    assert dsa.index_topk_workspace(lay, 64) > cap
    Q, K, W = (t.to("cuda:0") for t in (b.Q, b.K, b.W))
    with pytest.raises(dsa.DsaError) as e:
        dsa.index_topk_static(lay, Q, K, W, 64)
    assert e.value.status == 3
