"""GPU parity of PIVOT (Reuse / Refine) and HISA against the oracle.

Both methods are two-stage.  The first stage (PIVOT candidates, HISA kept
blocks) is compared with the oracle's under the same rule as the final
indices; the second stage is compared with the oracle's second stage run on
the GPU's own first-stage result (identical when the first stages agree).
Integer-valued inputs with power-of-two group sizes keep every proxy, pooled
key and score exact, so those cases are compared exactly.
"""
import numpy as np
import pytest

import oracle
import workloads
from parity import check_exact_sets, check_tolerance_row
from gpu_util import Dev, ascending_packed

pytestmark = pytest.mark.gpu


def group_rows(b, G):
    """Oracle output row of each query (groups are padded to G rows)."""
    rows = []
    qo = b.q_offsets.tolist()
    g0 = 0
    for s in range(b.num_seqs):
        nq = qo[s + 1] - qo[s]
        for j in range(nq):
            rows.append((g0 + j // G) * G + j % G)
        g0 += (nq + G - 1) // G
    return np.array(rows, dtype=np.int64)


# ------------------------------------------------------------------ PIVOT

@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("G,C,k", [(16, 256, 64), (4, 64, 64), (1, 64, 64)])
def test_pivot_integer_exact(mode, G, C, k):
    b = workloads.tiny_integer(seed=5, T=512, H=4, d=32, k=k)
    idx, cand = Dev(b).pivot(k, G, C, mode)
    ref = oracle.pivot(b, G, C, k)
    ascending_packed(cand)
    check_exact_sets(cand, ref["cand"], "cand")
    r = group_rows(b, G)
    check_exact_sets(idx, (ref["reuse_idx"] if mode == 0 else ref["refine_idx"])[r], "idx")


@pytest.mark.parametrize("mode", [0, 1])
def test_pivot_ragged_integer_exact(mode):
    b = workloads.ragged(7, [37, 64, 5], [37, 200, 90], H=4, d=32, k=16, integer=True)
    G, C, k = 8, 40, 16
    idx, cand = Dev(b).pivot(k, G, C, mode)
    ref = oracle.pivot(b, G, C, k)
    check_exact_sets(cand, ref["cand"], "cand")
    r = group_rows(b, G)
    check_exact_sets(idx, (ref["reuse_idx"] if mode == 0 else ref["refine_idx"])[r], "idx")


@pytest.mark.parametrize("mode", [0, 1])
def test_pivot_random_positions_exact(mode):
    """Queries of a group at scattered positions: Reuse serves some from the group's shared list and
    ranks the rest one by one; both must equal the oracle exactly."""
    b = workloads.ragged(41, [40, 24, 9], [300, 150, 64], H=4, d=32, k=24, integer=True, pos_mode="random")
    G, C, k = 8, 64, 24
    idx, cand = Dev(b).pivot(k, G, C, mode)
    ref = oracle.pivot(b, G, C, k)
    check_exact_sets(cand, ref["cand"], "cand")
    check_exact_sets(idx, (ref["reuse_idx"] if mode == 0 else ref["refine_idx"])[group_rows(b, G)], "idx")


@pytest.mark.parametrize("case", ["tiny", "ragged_random", "long_groups"])
def test_pivot_reuse_without_candidate_list_exact(case):
    """Reuse with no candidate list asked for selects each group's list from the proxy row itself and
    builds candidate lists only for queries the list does not serve (scattered positions); integer
    inputs, exact against the oracle."""
    if case == "tiny":
        b, (G, C, k) = workloads.tiny_integer(seed=5, T=512, H=4, d=32, k=64), (16, 256, 64)
    elif case == "ragged_random":
        b, (G, C, k) = workloads.ragged(41, [40, 24, 9], [300, 150, 64], H=4, d=32, k=24, integer=True,
                                        pos_mode="random"), (8, 64, 24)
    else:
        b, (G, C, k) = workloads.tiny_integer(seed=9, T=2048, H=4, d=32, k=128), (16, 512, 128)
    idx = Dev(b).pivot_idx(k, G, C, 0)
    ref = oracle.pivot(b, G, C, k)
    check_exact_sets(idx, ref["reuse_idx"][group_rows(b, G)], "idx")


def _random_candidates(b, G, C, seed, bad_group=None):
    """Per group: a sorted random subset of its sequence's keys (some past its queries' positions), -1
    padded; with bad_group, that group's list has a descending pair in the middle."""
    rng = np.random.default_rng(seed)
    qo, ko = b.q_offsets.tolist(), b.k_offsets.tolist()
    rows = []
    for s in range(b.num_seqs):
        L = ko[s + 1] - ko[s]
        for _ in range((qo[s + 1] - qo[s] + G - 1) // G):
            n = int(rng.integers(0, min(C, L) + 1))
            row = np.full(C, -1, np.int32)
            row[:n] = np.sort(rng.choice(L, size=n, replace=False))
            rows.append(row)
    cand = np.stack(rows)
    if bad_group is not None:   # single-sequence batch: a 32-key list with its middle pair swapped
        cand[bad_group] = -1
        cand[bad_group, :32] = np.sort(rng.choice(ko[1] - ko[0], size=32, replace=False))
        cand[bad_group, 16], cand[bad_group, 17] = cand[bad_group, 17], cand[bad_group, 16]
    return cand


@pytest.mark.parametrize("seed,q_lens,k_lens,mode", [(50, [64], [64], "suffix"), (51, [24, 40], [300, 90], "random")])
def test_refine_on_supplied_candidates_exact(seed, q_lens, k_lens, mode):
    """Refine over the caller's candidate lists equals the oracle's Refine on the same lists (integer,
    exact), including queries with no eligible candidate."""
    import sparse_attention_indexer_04_b200 as dsa
    import torch
    b = workloads.ragged(seed, q_lens, k_lens, H=4, d=32, k=16, integer=True, pos_mode=mode)
    G, C, k = 8, 48, 16
    cand = _random_candidates(b, G, C, seed)
    d = Dev(b)
    ws = torch.empty(dsa.pivot_refine_candidates_workspace(d.lay, k, G, C), dtype=torch.uint8, device="cuda:0")
    idx = dsa.pivot_refine_candidates(d.lay, d.Q, d.K, d.W, k, G, torch.as_tensor(cand).cuda(), ws=ws)
    assert dsa.device_check(ws) == 0
    ref = oracle.pivot(b, G, C, k, ext_cand=cand)
    check_exact_sets(idx.cpu().numpy(), ref["refine_idx"][group_rows(b, G)], "idx")


def test_refine_on_supplied_candidates_reports_a_bad_list():
    """A list with a descending pair is used up to it and reported (status code 2); other groups are exact."""
    import sparse_attention_indexer_04_b200 as dsa
    import torch
    b = workloads.tiny_integer(seed=52, T=256, H=4, d=32, k=16)
    G, C, k = 8, 64, 16
    cand = _random_candidates(b, G, C, 52, bad_group=5)
    d = Dev(b)
    ws = torch.empty(dsa.pivot_refine_candidates_workspace(d.lay, k, G, C), dtype=torch.uint8, device="cuda:0")
    idx = dsa.pivot_refine_candidates(d.lay, d.Q, d.K, d.W, k, G, torch.as_tensor(cand).cuda(), ws=ws).cpu().numpy()
    assert dsa.device_check(ws) == 2
    good = cand.copy()
    good[5, 17:] = -1                           # the usable prefix: up to the larger of the swapped pair
    ref = oracle.pivot(b, G, C, k, ext_cand=good)
    check_exact_sets(idx, ref["refine_idx"][group_rows(b, G)], "idx")


def test_pivot_reuse_long_groups_exact():
    """Reuse over a long prefill: groups of 16 consecutive queries, each query dropping up to 15 of the
    group's k + 15 best candidates; integer inputs with many ties, exact against the oracle."""
    b = workloads.tiny_integer(seed=9, T=2048, H=4, d=32, k=128)
    G, C, k = 16, 512, 128
    idx, cand = Dev(b).pivot(k, G, C, 0)
    ref = oracle.pivot(b, G, C, k)
    check_exact_sets(cand, ref["cand"], "cand")
    check_exact_sets(idx, ref["reuse_idx"][group_rows(b, G)], "idx")


def check_pivot_bf16(b, G, C, k, mode, groups=None, gpu=None):
    """bf16 PIVOT against the oracle: stage 1 (candidates) under the tolerance rule, stage 2 against the
    oracle's second stage on the GPU's own candidates.  `groups`: check only these groups (global group
    indices of a single-sequence batch); `gpu`: (idx, cand) already computed."""
    idx, cand = gpu if gpu is not None else Dev(b).pivot(k, G, C, mode)
    sel = list(range(cand.shape[0])) if groups is None else list(groups)
    own = oracle.pivot(b, G, C, k, groups=sel)                      # the oracle's own two stages
    ext = oracle.pivot(b, G, C, k, groups=sel, ext_cand=cand[sel])  # its second stage on the GPU's candidates
    gc = cand[sel].copy()
    ascending_packed(gc)
    # stage 1: candidate sets under the rule, scored by the oracle's proxy
    for i, g in enumerate(sel):
        sc = {}
        for src in (own, ext):
            v = src["cand"][i] >= 0
            sc.update(zip(src["cand"][i][v].tolist(), src["cand_score"][i][v].tolist()))
        rms = float(np.sqrt(np.mean(own["cand_score"][i][own["cand"][i] >= 0] ** 2)))
        msg = check_tolerance_row(gc[i], own["cand"][i], lambda ix: np.array([sc[x] for x in ix]), rms)
        assert msg is None, f"group {g} candidates: {msg}"
    # stage 2: each query against the oracle's second stage on the same candidates
    rows = group_rows(b, G)
    pos = {g: i for i, g in enumerate(sel)}
    for t in range(b.n_q):
        g = rows[t] // G
        if g not in pos:
            continue
        i, j = pos[g], rows[t] % G
        v = (ext["cand"][i] >= 0) & (ext["cand"][i] <= int(b.q_pos[t]))
        elig = ext["cand"][i][v]
        if mode == 0:
            prox = dict(zip(elig.tolist(), ext["cand_score"][i][v].tolist()))
            score_of = lambda ix, d=prox: np.array([d[x] for x in ix])
            ref_row = ext["reuse_idx"][i * G + j]
        else:
            own_sc = dict(zip(elig.tolist(), oracle.pair_scores(b, [t] * elig.size, elig).tolist()))
            score_of = lambda ix, d=own_sc: np.array([d[x] for x in ix])
            ref_row = ext["refine_idx"][i * G + j]
        fin = score_of(elig) if elig.size else np.zeros(1)
        rms = float(np.sqrt(np.mean(fin ** 2)))
        msg = check_tolerance_row(idx[t], ref_row, score_of, rms)
        assert msg is None, f"query {t}: {msg}"


@pytest.mark.parametrize("mode", [0, 1])
def test_pivot_bf16_small(mode):
    b = workloads.dense_prefill(seed=31, T=600, H=64, d=128, k=64)
    check_pivot_bf16(b, G=16, C=256, k=64, mode=mode)


@pytest.mark.parametrize("mode", [0, 1])
def test_pivot_decode_groups_are_mtp_steps(mode):
    """Decode: a group is the MTP queries of one step (group size = queries per sequence)."""
    b = workloads.dense_decode(seed=32, B=4, L=2000, n_mtp=2, H=64, d=128, k=128)
    check_pivot_bf16(b, G=2, C=512, k=128, mode=mode)


def test_full_size_pivot_128k_sampled_groups():
    """PIVOT at 128K (G = 16, C = 8192, k = 2048): the whole batch on the GPU in both modes; sampled
    groups (early ones whose prefix is shorter than C, middle and last) checked against the oracle."""
    b = workloads.pivot_prefill(seed=3)
    G, C, k = 16, 8192, 2048
    # 64 groups: the first few (prefix shorter than C), 59 more spread evenly over the sequence, the last two
    groups = sorted(set([0, 1, 3, 8190, 8191] + np.linspace(0, 8191, 61).astype(int).tolist()))
    assert len(groups) >= 64
    dev = Dev(b)
    reuse = dev.pivot(k, G, C, 0)
    refine = dev.pivot(k, G, C, 1)
    assert np.array_equal(reuse[1], refine[1])            # both modes share the candidate stage
    # Reuse with no candidate list asked for: the same indices, row for row
    assert np.array_equal(dev.pivot_idx(k, G, C, 0), reuse[0])
    check_pivot_bf16(b, G, C, k, 0, groups=groups, gpu=reuse)
    check_pivot_bf16(b, G, C, k, 1, groups=groups, gpu=refine)


# ------------------------------------------------------------------- HISA

def test_hisa_pool_integer_exact():
    """Integer keys: the block sums are exact in fp32, so each pooled key is the exact mean rounded once
    to fp32 (full blocks of 64 keys are exact; the partial last blocks hold 40 and 44 keys)."""
    b = workloads.ragged(8, [1, 1], [1000, 300], H=4, d=32, k=8, integer=True)
    _, _, pooled = Dev(b).hisa(8, 64, 4)
    ref = oracle.hisa_pool(b, 64)
    assert np.array_equal(pooled, ref.astype(np.float32))
    full = [j for j in range(ref.shape[0]) if j not in (15, 15 + 5)]
    assert np.array_equal(pooled[full].astype(np.float64), ref[full])


@pytest.mark.parametrize("B,keep", [(64, 3), (128, 1), (64, 40), (128, 4), (256, 2)])
def test_hisa_integer_exact(B, keep):
    b = workloads.ragged(9, [3, 2, 4], [1500, 700, 129], H=4, d=32, k=100, integer=True, pos_mode="random")
    idx, kept, _ = Dev(b).hisa(100, B, keep)
    ref = oracle.hisa(b, B, keep, 100)
    check_exact_sets(kept, ref["kept"], "kept")
    check_exact_sets(idx, ref["idx"], "idx")


def test_hisa_many_sequences_exact():
    """More sequences than the one-pass set-up takes (480): the step falls back to the staged path
    (CUDA-core block scores, streaming selects); 490 one-query sequences, integer inputs, exact."""
    lens = [200 + 37 * (i % 13) for i in range(490)]
    b = workloads.ragged(12, [1] * 490, lens, H=4, d=32, k=40, integer=True, pos_mode="random")
    idx, kept, _ = Dev(b).hisa(40, 64, 2)
    ref = oracle.hisa(b, 64, 2, 40)
    check_exact_sets(kept, ref["kept"], "kept")
    check_exact_sets(idx, ref["idx"], "idx")


def test_hisa_prefill_exact():
    """HISA in prefill (every position of a sequence is a query: the block filter runs per query over
    its own causal prefix); integer inputs, exact kept blocks and indices."""
    b = workloads.tiny_integer(seed=10, T=1500, H=4, d=32, k=96)
    idx, kept, _ = Dev(b).hisa(96, 64, 5)
    ref = oracle.hisa(b, 64, 5, 96)
    check_exact_sets(kept, ref["kept"], "kept")
    check_exact_sets(idx, ref["idx"], "idx")


def check_hisa_bf16(b, k, B, keep):
    idx, kept, pooled = Dev(b).hisa(k, B, keep)
    ascending_packed(kept)
    own = oracle.hisa(b, B, keep, k)
    for t in range(b.n_q):
        bs = own["block_scores"][t]
        mid = np.nonzero(~np.isnan(bs))[0]
        rms = float(np.sqrt(np.mean(bs[mid] ** 2))) if mid.size else 0.0
        strip = lambda r: r[(r >= 0)][1:-1] if (r >= 0).sum() > 1 else r[:0]
        gk, ok = kept[t], own["kept"][t]
        if mid.size:
            g_mid = np.concatenate([strip(gk), -np.ones(keep + 2, np.int32)])[:keep]
            o_mid = np.concatenate([strip(ok), -np.ones(keep + 2, np.int32)])[:keep]
            msg = check_tolerance_row(g_mid, o_mid, lambda ix: bs[ix], rms)
            assert msg is None, f"row {t} kept blocks: {msg}"
    ext = oracle.hisa(b, B, keep, k, ext_kept=kept)
    for t in range(b.n_q):
        cols = []
        p = int(b.q_pos[t])
        for blk in kept[t][kept[t] >= 0]:
            cols.extend(range(blk * B, min(blk * B + B, p + 1)))
        sc = oracle.pair_scores(b, [t] * len(cols), cols)
        d = dict(zip(cols, sc))
        rms = float(np.sqrt(np.mean(sc ** 2))) if len(cols) else 0.0
        msg = check_tolerance_row(idx[t], ext["idx"][t], lambda ix: np.array([d[x] for x in ix]), rms)
        assert msg is None, f"row {t}: {msg}"


def test_hisa_bf16_needles():
    b = workloads.hisa_decode(seed=41, B=2, L=40000, n_mtp=2, H=64, d=128, k=512, block=128, keep=16,
                              n_needles=6)
    check_hisa_bf16(b, 512, 128, 16)


@pytest.mark.parametrize("keep", [40, 100])
def test_hisa_bf16_long_token_rows(keep):
    """Token rows of 5376 and 13056 columns (40 and 100 kept middle blocks of 128): the longer
    register top-k shapes."""
    b = workloads.hisa_decode(seed=43, B=2, L=20000, n_mtp=2, H=64, d=128, k=2048, block=128, keep=keep,
                              n_needles=4)
    check_hisa_bf16(b, 2048, 128, keep)


def test_full_size_hisa_256k():
    """HISA decode at 256K: 4 sequences, 2 queries, H=64, d=128, k=2048, block 128, keep 64 (+2)."""
    b = workloads.hisa_decode(seed=4)
    check_hisa_bf16(b, 2048, 128, 64)
