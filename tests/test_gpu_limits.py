"""Parity at the edges of the supported shapes (integer inputs, exact against the oracle): the smallest
and largest k, the largest PIVOT group and candidate count, the largest HISA block and kept count."""
import numpy as np
import pytest

import oracle
import workloads
from parity import check_exact_sets
from gpu_util import Dev, ascending_packed

pytestmark = pytest.mark.gpu


def test_k_is_one():
    b = workloads.tiny_integer(seed=70, T=700, H=4, d=32, k=1)
    idx = Dev(b).topk(1)
    check_exact_sets(idx, oracle.dense(b, k=1)["idx"])


def test_largest_k_over_a_long_row():
    """k = 16384 (the largest supported) over rows of ~20000 keys: the candidate buffer is clamped to the
    shared memory left by the row's bitmaps; every row still ranks exactly."""
    b = workloads.ragged(71, [3], [20000], H=4, d=32, k=16384, integer=True)
    idx = Dev(b).topk(16384)
    ascending_packed(idx)
    check_exact_sets(idx, oracle.dense(b, k=16384)["idx"])


def test_largest_pivot_group_and_candidate_count():
    b = workloads.tiny_integer(seed=72, T=300, H=4, d=32, k=32)
    G, C, k = 64, 16384, 32
    for mode in (0, 1):
        idx, cand = Dev(b).pivot(k, G, C, mode)
        ref = oracle.pivot(b, G, C, k)
        check_exact_sets(cand, ref["cand"], "cand")
        rows = np.arange(b.n_q)                      # one sequence: query t is output row t
        check_exact_sets(idx, (ref["reuse_idx"] if mode == 0 else ref["refine_idx"])[rows], "idx")


def test_largest_hisa_block_and_keep():
    b = workloads.ragged(73, [2, 3], [70000, 2000], H=4, d=32, k=64, integer=True, pos_mode="random")
    idx, kept, _ = Dev(b).hisa(64, 256, 256)
    ref = oracle.hisa(b, 256, 256, 64)
    check_exact_sets(kept, ref["kept"], "kept")
    check_exact_sets(idx, ref["idx"], "idx")


def test_longest_supported_row():
    """Rows of 757,000 keys, just under the longest the selection's shared memory holds (two column
    bitmaps next to the sample and a candidate buffer clamped to 256 entries): exact all the same."""
    b = workloads.ragged(74, [2], [757000], H=4, d=32, k=64, integer=True)
    idx = Dev(b).topk(64)
    ascending_packed(idx)
    check_exact_sets(idx, oracle.dense(b, k=64)["idx"])
