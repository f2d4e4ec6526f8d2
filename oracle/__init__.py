"""ctypes binding of the fp64 CPU oracle (oracle/oracle.c).

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's CPU
baseline import this package.  The CUDA library and its Python binding never
do.  Inputs are the CPU tensors of a ``workloads.Batch``; bf16 tensors are
handed over as their bit patterns and decoded inside the C code.

Parity pins for every function here live in tests/test_oracle_pins.py; none
of the functions is unpinned.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from .build import build

_lib = None
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.orc_round_bf16.restype = ctypes.c_double
        _lib.orc_round_bf16.argtypes = [ctypes.c_double]
        _lib.orc_pivot_num_groups.restype = ctypes.c_int64
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _bits(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _i32(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


class _Common:
    def __init__(self, batch):
        self.Q = _bits(batch.Q)
        self.K = _bits(batch.K)
        self.W = np.ascontiguousarray(batch.W.numpy().astype(np.float32))
        self.q_off = _i32(batch.q_offsets)
        self.k_off = _i32(batch.k_offsets)
        self.q_pos = _i32(batch.q_pos)
        self.H, self.d = batch.H, batch.d
        self.n_seqs = batch.num_seqs


def round_bf16(x: float) -> float:
    """Nearest bf16 value of a double, ties to even."""
    return lib().orc_round_bf16(float(x))


def dense(batch, rows=None, k=None, want_all=False, threads=None):
    """Dense indexer on the listed query rows.

    Returns dict: idx [n,k] int32 (ranking order, -1 padded), top [n,k] fp64,
    n_elig [n] int32 and, with want_all, all [n, max_len] fp64 (-inf where ineligible).
    """
    c = _Common(batch)
    rows = _i32(range(batch.n_q) if rows is None else rows)
    n = rows.size
    k = int(batch.params.get("k", 1) if k is None else k)
    ld = max(batch.seq_lens()) if batch.num_seqs else 0
    idx = np.empty((n, k), np.int32)
    top = np.empty((n, k), np.float64)
    n_elig = np.empty(n, np.int32)
    allsc = np.empty((n, max(ld, 1)), np.float64) if want_all else None
    lib().orc_dense(_p(c.Q), _p(c.K), _p(c.W), c.H, c.d, c.n_seqs, _p(c.q_off), _p(c.k_off),
                    _p(c.q_pos), n, _p(rows), k, _p(idx), _p(top), _p(allsc), ctypes.c_int64(ld),
                    _p(n_elig), threads or default_threads())
    out = dict(idx=idx, top=top, n_elig=n_elig)
    if want_all:
        out["all"] = allsc[:, :ld]
    return out


def pair_scores(batch, rows, keys, threads=None):
    """Indexer score of each (query row, sequence-local key) pair, in fp64."""
    c = _Common(batch)
    rows, keys = _i32(rows), _i32(keys)
    out = np.empty(rows.size, np.float64)
    lib().orc_pair_scores(_p(c.Q), _p(c.K), _p(c.W), c.H, c.d, c.n_seqs, _p(c.q_off), _p(c.k_off),
                          ctypes.c_int64(rows.size), _p(rows), _p(keys), _p(out),
                          threads or default_threads())
    return out


def pivot_num_groups(batch, G):
    return int(lib().orc_pivot_num_groups(batch.num_seqs, _p(_i32(batch.q_offsets)), int(G)))


def pivot(batch, G, C, k, groups=None, ext_cand=None, threads=None):
    """PIVOT on the listed groups.  Query rows of the i-th listed group are output rows i*G .. i*G+G-1."""
    c = _Common(batch)
    if groups is None:
        groups = range(pivot_num_groups(batch, G))
    groups = _i32(groups)
    n = groups.size
    cand = np.empty((n, C), np.int32)
    cand_score = np.empty((n, C), np.float64)
    reuse_idx = np.empty((n * G, k), np.int32)
    reuse_score = np.empty((n * G, k), np.float64)
    refine_idx = np.empty((n * G, k), np.int32)
    refine_score = np.empty((n * G, k), np.float64)
    pq = np.empty((n, c.H * c.d), np.float64)
    pw = np.empty((n, c.H), np.float64)
    ext = None if ext_cand is None else _i32(ext_cand).reshape(n, C)
    lib().orc_pivot(_p(c.Q), _p(c.K), _p(c.W), c.H, c.d, c.n_seqs, _p(c.q_off), _p(c.k_off),
                    _p(c.q_pos), int(G), int(C), int(k), n, _p(groups), _p(ext), _p(cand),
                    _p(cand_score), _p(reuse_idx), _p(reuse_score), _p(refine_idx), _p(refine_score),
                    _p(pq), _p(pw), threads or default_threads())
    return dict(cand=cand, cand_score=cand_score, reuse_idx=reuse_idx, reuse_score=reuse_score,
                refine_idx=refine_idx, refine_score=refine_score,
                proxy_q=pq.reshape(n, c.H, c.d), proxy_w=pw)


def hisa_num_blocks(batch, B):
    return sum((L + B - 1) // B for L in batch.seq_lens())


def hisa_pool(batch, B):
    """Mean-pooled block keys of every sequence, stacked: [sum_b ceil(L_b/B), d] fp64."""
    c = _Common(batch)
    out = np.empty((hisa_num_blocks(batch, B), c.d), np.float64)
    lib().orc_hisa_pool(_p(c.K), c.d, c.n_seqs, _p(c.k_off), int(B), _p(out))
    return out


def hisa(batch, B, keep, k, rows=None, pooled=None, ext_kept=None, threads=None):
    """HISA on the listed query rows.

    Returns dict: kept [n, keep+2] (ascending, -1 padded), block_scores
    [n, max_blocks] (NaN except middle blocks), idx / top [n, k].
    """
    c = _Common(batch)
    rows = _i32(range(batch.n_q) if rows is None else rows)
    n = rows.size
    if pooled is None:
        pooled = hisa_pool(batch, B)
    pooled = np.ascontiguousarray(pooled, dtype=np.float64)
    max_blocks = max((L + B - 1) // B for L in batch.seq_lens())
    kept = np.empty((n, keep + 2), np.int32)
    bs = np.empty((n, max_blocks), np.float64)
    idx = np.empty((n, k), np.int32)
    top = np.empty((n, k), np.float64)
    ext = None if ext_kept is None else _i32(ext_kept).reshape(n, keep + 2)
    lib().orc_hisa(_p(c.Q), _p(c.K), _p(c.W), _p(pooled), c.H, c.d, c.n_seqs, _p(c.q_off),
                   _p(c.k_off), _p(c.q_pos), int(B), int(keep), int(k), n, _p(rows), _p(ext),
                   _p(kept), _p(bs), ctypes.c_int64(max_blocks), _p(idx), _p(top),
                   threads or default_threads())
    return dict(kept=kept, block_scores=bs, idx=idx, top=top)


def layer_sources(n_layers, retain_every, lag):
    """For each of n_layers consecutive layers, the layer whose indexer made its selection, stepping
    through the layers as the pages describe.  IndexCache (MLI abstract; related-paper list of the
    PIVOT page): one layer in `retain_every` is "full" and runs its own indexer, starting with the
    first; a "shared" layer reuses the top-k of the nearest full layer before it.  MLI (MLI
    abstract), lag = 1: a layer attends over the selection the previous layer's indexer made, so its
    own indexer can run beside its attention; the first layer has no predecessor and uses its own."""
    src = []
    last_full = None
    prev_sel = None
    for layer in range(n_layers):
        if layer % retain_every == 0:
            last_full = layer
        own_sel = last_full                     # what this layer's (possibly reused) indexer provides
        src.append(prev_sel if lag and layer > 0 else own_sel)
        prev_sel = own_sel
    return src


def layer_topk(batches, k, retain_every, lag, threads=None):
    """Selections of consecutive layers (one workloads.Batch per layer, same layout): the dense
    top-k of each layer's source layer (layer_sources)."""
    src = layer_sources(len(batches), retain_every, lag)
    own = {}
    out = []
    for s in src:
        if s not in own:
            own[s] = dense(batches[s], k=k, threads=threads)["idx"]
        out.append(own[s])
    return out
