"""Seeded synthetic inputs for the DSA lightning-indexer workloads.

This module only draws random numbers and lays them out; it holds none of the
indexer's arithmetic (no scoring, no selection, no pooling, no proxies).  Both
the CPU oracle (``oracle/``) and the CUDA library are fed from the tensors it
returns, so the two sides always see the same bf16 / fp32 values.

Shapes follow the workloads the pages describe (DeepSeek-V3.2-style indexer:
64 heads of dimension 128, k = 2048, long contexts) and stand in for the
LongBench / RULER / needle-in-a-haystack inputs the pages evaluate on; no item
of those suites is used.  Every tensor is created on the CPU from a
``torch.Generator`` seeded explicitly, in fp32, then rounded to bf16 with
round-to-nearest-even (``Tensor.to(torch.bfloat16)``).

Layout of a batch (all CPU tensors):
  Q         [n_q, H, d]  bf16   query rows of every sequence, concatenated
  K         [n_k, d]     bf16   one key per token, shared by all heads
  W         [n_q, H]     fp32   per-query, per-head weights
  q_offsets [B+1]        int32  rows q_offsets[b] .. q_offsets[b+1]-1 belong to sequence b
  k_offsets [B+1]        int32  key rows of sequence b
  q_pos     [n_q]        int32  sequence-local position of each query (causal limit)
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass
class Batch:
    Q: torch.Tensor
    K: torch.Tensor
    W: torch.Tensor
    q_offsets: torch.Tensor
    k_offsets: torch.Tensor
    q_pos: torch.Tensor
    params: dict = field(default_factory=dict)
    name: str = ""

    @property
    def n_q(self) -> int:
        return int(self.Q.shape[0])

    @property
    def H(self) -> int:
        return int(self.Q.shape[1])

    @property
    def d(self) -> int:
        return int(self.Q.shape[2])

    @property
    def num_seqs(self) -> int:
        return int(self.q_offsets.numel() - 1)

    def seq_lens(self):
        ko = self.k_offsets.tolist()
        return [ko[i + 1] - ko[i] for i in range(len(ko) - 1)]

    def eligible_pairs(self) -> int:
        """Number of (query, key) pairs with key position <= query position."""
        qo, ko, pos = self.q_offsets.tolist(), self.k_offsets.tolist(), self.q_pos
        total = 0
        for b in range(len(qo) - 1):
            L = ko[b + 1] - ko[b]
            p = pos[qo[b]:qo[b + 1]].to(torch.int64)
            total += int(torch.clamp(torch.minimum(p + 1, torch.tensor(L)), min=0).sum())
        return total


def _offsets(lengths):
    out = [0]
    for n in lengths:
        out.append(out[-1] + int(n))
    return torch.tensor(out, dtype=torch.int32)


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.bfloat16)


def _randn(g, *shape):
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def tiny_integer(seed: int = 0, T: int = 512, H: int = 4, d: int = 32, k: int = 64,
                 signed_w: bool = False) -> Batch:
    """Integer-valued single-sequence prefill (T = L, causal).

    Q, K uniform integers in [-3, 3]; w uniform over {0.25, 0.5, 1, 2}
    (or over {-2, -1, -0.5, 0.5, 1, 2} with ``signed_w``).  Every product and
    every partial sum is a multiple of 0.25 below 2**24 in magnitude, so the
    scores are exact in fp32 whatever the summation order.
    """
    g = torch.Generator().manual_seed(seed)
    Q = torch.randint(-3, 4, (T, H, d), generator=g).to(torch.float32)
    K = torch.randint(-3, 4, (T, d), generator=g).to(torch.float32)
    choices = torch.tensor([-2.0, -1.0, -0.5, 0.5, 1.0, 2.0] if signed_w else [0.25, 0.5, 1.0, 2.0])
    W = choices[torch.randint(0, choices.numel(), (T, H), generator=g)]
    return Batch(_bf16(Q), _bf16(K), W.contiguous(), _offsets([T]), _offsets([T]),
                 torch.arange(T, dtype=torch.int32), dict(k=k), f"tiny_int_T{T}_H{H}_d{d}")


def _rank_r_queries(g, T, H, d, rank=8, rho=0.99, chunk=4096):
    """Q[t,h] = 0.6 N(0,I) + (0.8/sqrt(rank)) sum_r a_r(t) U_r[h].

    U_r[h] ~ N(0, I) is fixed; a_r(t) is an AR(1) process along t with
    coefficient rho and unit stationary variance, so neighbouring queries share
    a slowly varying low-rank component (the pages observe that nearby queries
    select overlapping top-k sets).
    """
    U = _randn(g, rank, H * d)
    a = torch.empty(T, rank)
    a[0] = _randn(g, rank)
    innov = _randn(g, T, rank) * math.sqrt(1.0 - rho * rho)
    for t in range(1, T):
        a[t] = rho * a[t - 1] + innov[t]
    Q = torch.empty(T, H, d, dtype=torch.bfloat16)
    scale = 0.8 / math.sqrt(rank)
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        x = 0.6 * _randn(g, t1 - t0, H * d) + scale * (a[t0:t1] @ U)
        Q[t0:t1] = _bf16(x.view(t1 - t0, H, d))
    return Q


def dense_prefill(seed: int = 2, T: int = 32768, H: int = 64, d: int = 128, k: int = 2048,
                  rank: int = 8, rho: float = 0.99) -> Batch:
    """Single-sequence causal prefill, T = L: keys N(0,1), w ~ N(0,1)/8, rank-`rank` shared query part."""
    g = torch.Generator().manual_seed(seed)
    K = _bf16(_randn(g, T, d))
    W = _randn(g, T, H) / 8.0
    Q = _rank_r_queries(g, T, H, d, rank, rho)
    return Batch(Q, K, W, _offsets([T]), _offsets([T]), torch.arange(T, dtype=torch.int32),
                 dict(k=k), f"dense_prefill_T{T}_H{H}_d{d}")


def pivot_prefill(seed: int = 3, T: int = 131072, H: int = 64, d: int = 128, k: int = 2048,
                  group: int = 16, n_cand: int = 8192) -> Batch:
    """Inputs drawn as ``dense_prefill`` at length T, with PIVOT's group size and candidate count."""
    b = dense_prefill(seed, T, H, d, k)
    b.params.update(group=group, n_cand=n_cand)
    b.name = f"pivot_prefill_T{T}_G{group}_C{n_cand}"
    return b


def dense_decode(seed: int = 1, B: int = 16, L: int = 32768, n_mtp: int = 2, H: int = 64,
                 d: int = 128, k: int = 2048) -> Batch:
    """Batched decode: B caches of L keys each, n_mtp queries per sequence at positions L-n_mtp .. L-1."""
    g = torch.Generator().manual_seed(seed)
    K = _bf16(_randn(g, B * L, d))
    Q = _bf16(_randn(g, B * n_mtp, H, d))
    W = _randn(g, B * n_mtp, H) / 8.0
    pos = torch.tensor([L - n_mtp + j for _ in range(B) for j in range(n_mtp)], dtype=torch.int32)
    return Batch(Q, K, W, _offsets([n_mtp] * B), _offsets([L] * B), pos, dict(k=k),
                 f"dense_decode_B{B}_L{L}_mtp{n_mtp}")


def hisa_decode(seed: int = 4, B: int = 4, L: int = 262144, n_mtp: int = 2, H: int = 64,
                d: int = 128, k: int = 2048, block: int = 128, keep: int = 64,
                n_needles: int = 8, span: int = 64) -> Batch:
    """Batched decode with planted needle spans.

    Keys are N(0, I) except `n_needles` spans of `span` tokens per sequence,
    placed at seeded offsets that are not multiples of the block size, where
    k_s = u + 0.5 N(0, I) with u ~ N(0, I) fixed per sequence.  Queries are
    q[t,h] = N(0, I) + 0.25 sign(w[t,h]) u, w ~ N(0,1)/8, so heads with w > 0
    score the needles high.  ``params['needles']`` lists each span's
    (sequence, start) for recall statistics.
    """
    g = torch.Generator().manual_seed(seed)
    Kf = _randn(g, B * L, d)
    W = _randn(g, B * n_mtp, H) / 8.0
    Qf = _randn(g, B * n_mtp, H, d)
    needles = []
    for b in range(B):
        u = _randn(g, d)
        starts = set()
        while len(starts) < n_needles:
            s = int(torch.randint(block, L - block - span, (1,), generator=g))
            if s % block == 0 or any(abs(s - o) < span for o in starts):
                continue
            starts.add(s)
        for s in sorted(starts):
            Kf[b * L + s: b * L + s + span] = u + 0.5 * _randn(g, span, d)
            needles.append((b, s))
        for j in range(n_mtp):
            t = b * n_mtp + j
            Qf[t] += 0.25 * torch.sign(W[t]).unsqueeze(1) * u.unsqueeze(0)
    pos = torch.tensor([L - n_mtp + j for _ in range(B) for j in range(n_mtp)], dtype=torch.int32)
    return Batch(_bf16(Qf), _bf16(Kf), W, _offsets([n_mtp] * B), _offsets([L] * B), pos,
                 dict(k=k, block=block, keep=keep, needles=needles, span=span),
                 f"hisa_decode_B{B}_L{L}")


def ragged(seed: int, q_lens, k_lens, H: int = 4, d: int = 32, k: int = 16,
           integer: bool = False, pos_mode: str = "suffix") -> Batch:
    """Ragged multi-sequence batch for edge cases.

    Sequence b has k_lens[b] keys and q_lens[b] queries.  pos_mode "suffix"
    puts the queries at the last q_lens[b] positions (prefill when
    q_len == k_len, decode when q_len is small); "random" draws positions
    uniformly in [-1, k_len] (out-of-range positions exercise the clamp).
    """
    g = torch.Generator().manual_seed(seed)
    n_q, n_k = sum(q_lens), sum(k_lens)
    if integer:
        Q = torch.randint(-3, 4, (n_q, H, d), generator=g).float()
        K = torch.randint(-3, 4, (n_k, d), generator=g).float()
        W = torch.tensor([0.25, 0.5, 1.0, 2.0])[torch.randint(0, 4, (n_q, H), generator=g)]
    else:
        Q, K, W = _randn(g, n_q, H, d), _randn(g, n_k, d), _randn(g, n_q, H) / 8.0
    pos = []
    for nq, nk in zip(q_lens, k_lens):
        if pos_mode == "suffix":
            pos += [nk - nq + j for j in range(nq)]
        else:
            pos += torch.randint(-1, nk + 1, (nq,), generator=g).tolist()
    return Batch(_bf16(Q), _bf16(K), W.contiguous(), _offsets(q_lens), _offsets(k_lens),
                 torch.tensor(pos, dtype=torch.int32), dict(k=k), f"ragged_{seed}")


def stratified_rows(n_rows: int, n_sample: int = 1024, head: int = 16, tail: int = 64, seed: int = 12345):
    """Deterministic row sample: rows 0..head-1, the last `tail` rows, and evenly spread rows between."""
    if n_rows <= n_sample:
        return list(range(n_rows))
    rows = set(range(min(head, n_rows))) | set(range(max(0, n_rows - tail), n_rows))
    g = torch.Generator().manual_seed(seed)
    rest = n_sample - len(rows)
    edges = torch.linspace(head, n_rows - tail, rest + 1).long().tolist()
    for i in range(rest):
        lo, hi = edges[i], max(edges[i] + 1, edges[i + 1])
        rows.add(int(torch.randint(lo, hi, (1,), generator=g)))
    return sorted(rows)
