"""GPU parity of the dense indexer (scores and top-k) against the oracle.

Integer-valued inputs: exact (fp32 scores bit-equal to the fp64 oracle,
index sets equal, ties to the lower index).  bf16 inputs: the tolerance rule
of tests/parity.py (relative 2e-3 of max(|k-th score|, row RMS)).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_exact_sets, check_scores_close, check_tolerance_rows
from gpu_util import Dev, ascending_packed

pytestmark = pytest.mark.gpu


def exact_topk(b, k):
    d = Dev(b)
    idx, sc = d.topk(k, want_scores=True)
    ref = oracle.dense(b, k=k, want_all=True)
    ascending_packed(idx)
    check_exact_sets(idx, ref["idx"])
    # returned scores: exactly the oracle's score of each returned index
    for t in range(b.n_q):
        v = idx[t] >= 0
        assert np.array_equal(sc[t][v].astype(np.float64), ref["all"][t][idx[t][v]]), t
        assert np.all(np.isnan(sc[t][~v]))
    return d, ref


def test_tiny_integer_prefill_exact():
    b = workloads.tiny_integer(seed=0, T=512, H=4, d=32, k=64)
    d, ref = exact_topk(b, 64)
    S = d.scores()
    assert np.array_equal(S.astype(np.float64), ref["all"])


def test_signed_weights_exact():
    exact_topk(workloads.tiny_integer(seed=1, T=300, H=4, d=32, k=40, signed_w=True), 40)


@pytest.mark.parametrize("H,dim", [(1, 32), (8, 64), (16, 128), (64, 32), (2, 128)])
def test_head_shapes_exact(H, dim):
    exact_topk(workloads.tiny_integer(seed=H + dim, T=260, H=H, d=dim, k=33), 33)


@pytest.mark.parametrize("seed,q_lens,k_lens,mode", [
    (10, [5, 1, 64], [300, 17, 129], "random"),
    (11, [200, 3], [200, 1000], "suffix"),
    (12, [1, 1, 1, 1], [1, 2, 130, 257], "suffix"),
    (13, [0, 40, 0], [10, 40, 5], "random"),
])
def test_ragged_batches_exact(seed, q_lens, k_lens, mode):
    exact_topk(workloads.ragged(seed, q_lens, k_lens, H=4, d=32, k=24, integer=True, pos_mode=mode), 24)


def test_k_larger_than_every_row():
    b = workloads.tiny_integer(seed=2, T=200, H=4, d=32, k=300)
    exact_topk(b, 300)


def test_all_equal_scores_take_lowest_indices():
    b = workloads.tiny_integer(seed=3, T=400, H=4, d=32, k=50)
    b.K = torch.ones_like(b.K)
    b.Q = torch.ones_like(b.Q)
    idx = Dev(b).topk(50)
    for t in range(b.n_q):
        n = min(50, t + 1)
        assert idx[t].tolist() == list(range(n)) + [-1] * (50 - n)


def test_empty_query_batch():
    b = workloads.ragged(4, [0], [10], H=4, d=32, k=8)
    d = Dev(b)
    assert d.topk(8).shape == (0, 8)


def test_bf16_prefill_tolerance():
    b = workloads.dense_prefill(seed=21, T=700, H=64, d=128, k=100)
    d = Dev(b)
    idx = d.topk(100)
    ascending_packed(idx)
    ref = oracle.dense(b, k=100, want_all=True)
    check_tolerance_rows(idx, ref["idx"], ref["all"])
    check_scores_close(d.scores(), ref["all"])


def test_bf16_decode_tolerance():
    b = workloads.dense_decode(seed=22, B=3, L=3000, n_mtp=2, H=64, d=128, k=256)
    d = Dev(b)
    idx = d.topk(256)
    ascending_packed(idx)
    ref = oracle.dense(b, k=256, want_all=True)
    check_tolerance_rows(idx, ref["idx"], ref["all"])


def test_full_size_decode_32k():
    """Dense decode, 16 sequences x 32K keys, 2 MTP queries each, H=64, d=128, k=2048: every row."""
    b = workloads.dense_decode(seed=1)
    idx = Dev(b).topk(2048)
    ascending_packed(idx)
    ref = oracle.dense(b, k=2048, want_all=True)
    check_tolerance_rows(idx, ref["idx"], ref["all"])


def test_full_size_decode_128k():
    """Dense decode, 16 sequences x 128K keys, 2 MTP queries each (the decode metric's size): every row."""
    b = workloads.dense_decode(seed=1, L=131072)
    idx = Dev(b).topk(2048)
    ascending_packed(idx)
    ref = oracle.dense(b, k=2048, want_all=True)
    check_tolerance_rows(idx, ref["idx"], ref["all"])


def test_full_size_prefill_32k_sampled_rows():
    """Dense prefill T = L = 32K, H=64, d=128, k=2048: the whole batch on the GPU, sampled rows checked."""
    b = workloads.dense_prefill(seed=2)
    idx = Dev(b).topk(2048)
    rows = workloads.stratified_rows(b.n_q, n_sample=1024, head=16, tail=64)   # rows 0-15, the last 64, the rest spread
    ref = oracle.dense(b, rows=rows, k=2048, want_all=True)
    ascending_packed(idx[rows])
    check_tolerance_rows(idx[rows], ref["idx"], ref["all"])
    # every row holds min(k, t+1) indices, all causal
    counts = (idx >= 0).sum(1)
    assert np.array_equal(counts, np.minimum(np.arange(b.n_q) + 1, 2048))
    assert np.all(idx.max(1) <= np.arange(b.n_q))


@pytest.mark.parametrize("n_rows", [2, 30, 300])
@pytest.mark.parametrize("sampled_high", [True, False])
def test_select_when_the_even_sample_misleads(sampled_high, n_rows):
    """The top-k picks a threshold from a sample of a long row: 2048 columns in 64 evenly spaced runs of
    32.  Keys that make exactly those columns score high (too few columns then pass the threshold) or
    low (too many pass) must still give the exact answer: integer inputs, compared exactly with the
    oracle.  Two rows take the split select (9 CTAs per row, sharing a global buffer), 30 rows the
    cluster select (4 CTAs per row as one cluster), 300 rows the one-CTA-per-row select."""
    L, k = 20000, 3000
    b = workloads.ragged(30, [n_rows], [L], H=1, d=32, k=k, integer=True)
    starts = ((np.arange(64, dtype=np.int64) * L) // 64) & ~31        # the sample of a row of n = L
    sampled = np.unique((starts[:, None] + np.arange(32)[None, :]).ravel())
    hi, lo = (3.0, 1.0) if sampled_high else (1.0, 3.0)
    K = np.full((L, 32), lo, np.float32)
    K[sampled] = hi
    K[::7, 0] += 1.0                       # some variation, many exact ties remain
    b.K = torch.as_tensor(K).to(torch.bfloat16)
    b.Q = torch.ones_like(b.Q)
    b.W = torch.ones_like(b.W)
    pos = np.full(n_rows, L - 1, np.int32)
    pos[0] = L - 2
    b.q_pos = torch.as_tensor(pos)
    exact_topk(b, k)


@pytest.mark.parametrize("seed,q_lens,k_lens,k,mode", [
    (40, [2, 1, 3], [9000, 20000, 4500], 1000, "suffix"),
    (41, [2, 2], [30000, 700], 2048, "random"),
    (42, [1] * 20, [5000 + 997 * i for i in range(20)], 512, "suffix"),
])
def test_few_long_rows_exact(seed, q_lens, k_lens, k, mode):
    """Few rows of many columns (decode): each row is ranked by several CTAs.  The first two cases
    (6 and 4 rows: 9 and 14 CTAs per row, more than a cluster of 8) take the split select, whose CTAs
    share one candidate buffer in global memory; the third (20 rows of up to ~24K columns: 7 CTAs
    per row) takes the cluster select, whose CTAs meet in the leader's shared memory.  Integer
    inputs (many ties across the CTAs' column chunks), a row shorter than k, clamped positions;
    exact against the oracle."""
    exact_topk(workloads.ragged(seed, q_lens, k_lens, H=4, d=32, k=k, integer=True, pos_mode=mode), k)


def test_cluster_select_short_rows_exact():
    """The cluster select (20 single-query rows, the longest of 16K columns or more: 7 CTAs per row)
    on rows that need no threshold: a row shorter than k (every column taken, -1 padding) and a row
    with k < n <= the candidate buffer (the whole row goes into the buffer), beside long rows.
    Integer inputs, exact against the oracle."""
    k_lens = [300, 3000] + [16384 + 1231 * i for i in range(18)]
    exact_topk(workloads.ragged(43, [1] * 20, k_lens, H=4, d=32, k=512, integer=True, pos_mode="suffix"), 512)


@pytest.mark.parametrize("make", [
    lambda: workloads.dense_prefill(seed=2),                                     # 8 row chunks, largest work first
    lambda: workloads.ragged(60, [5, 0, 64], [300, 17, 129], H=4, d=32, k=24),   # one chunk, ragged
    # 5 chunks of 2048 rows over three sequences with random positions: the work order is a
    # permutation of the row order and the three buffers rotate
    lambda: workloads.ragged(62, [3000, 2500, 4000], [3000, 6000, 4000], H=4, d=32, k=64, pos_mode="random"),
    lambda: workloads.dense_decode(seed=61, B=4, L=5000, n_mtp=2, H=64, d=128, k=256),
])
def test_host_memory_entry_matches_device_entry(make):
    """dsa_index_topk_host (inputs and indices in pinned host memory, copies overlapped with the work)
    returns exactly what dsa_index_topk returns on device copies of the same inputs."""
    import sparse_attention_indexer_04_b200 as dsa
    b = make()
    k = int(b.params["k"])
    d = Dev(b)
    ref = d.topk(k)
    hidx = torch.full((b.n_q, k), -7, dtype=torch.int32).pin_memory()
    ws = torch.empty(dsa.index_topk_host_workspace(d.lay, k), dtype=torch.uint8, device="cuda:0")
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    dsa.index_topk_host(d.lay, b.q_pos.to(torch.int32).contiguous().pin_memory(), b.Q.pin_memory(), b.K.pin_memory(),
                        b.W.contiguous().pin_memory(), k, hidx, ws, in_stream=s_in, out_stream=s_out)
    torch.cuda.current_stream().synchronize()
    assert dsa.device_check(ws) == 0
    assert np.array_equal(hidx.numpy(), ref)
