"""Cross-layer index reuse (dsa_index_layers) on the GPU against the oracle.

Each layer has its own integer-valued Q, K and W (exact scores), so the selection of every layer
must equal, bit for bit as index sets, the oracle's dense top-k of the layer whose indexer run it
takes (IndexCache: the nearest full layer; MLI: the previous layer's).  Layers that share a run
hold identical rows.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_indexer_04_b200 as dsa
import workloads
from gpu_util import ascending_packed
from parity import check_exact_sets

pytestmark = pytest.mark.gpu


def layer_inputs(n_layers, seed, T=300, H=4, d=32):
    bs = [workloads.tiny_integer(seed=seed + l, T=T, H=H, d=d, k=24) for l in range(n_layers)]
    dev = torch.device("cuda:0")
    lay = dsa.Layout.from_batch(bs[0], dev)   # every layer shares the layout
    Qs = [b.Q.to(dev) for b in bs]
    Ks = [b.K.to(dev) for b in bs]
    Ws = [b.W.to(dev) for b in bs]
    return bs, lay, Qs, Ks, Ws


@pytest.mark.parametrize("n_layers,r,lag", [(4, 2, 0), (6, 2, 1), (5, 1, 1), (3, 1, 0), (7, 3, 1)])
def test_layer_selections_match_the_oracle(n_layers, r, lag):
    bs, lay, Qs, Ks, Ws = layer_inputs(n_layers, seed=70 + 10 * n_layers + r + lag)
    side = torch.cuda.Stream()
    idx = dsa.index_layers(lay, Qs, Ks, Ws, 24, retain_every=r, lag=lag, side_stream=side)
    torch.cuda.current_stream().synchronize()
    want = oracle.layer_topk(bs, 24, r, lag)
    src = oracle.layer_sources(n_layers, r, lag)
    for l in range(n_layers):
        got = idx[l].cpu().numpy()
        ascending_packed(got)
        check_exact_sets(got, want[l], f"layer {l} (source {src[l]})")
        if src[l] != l and src[l] < n_layers:
            assert np.array_equal(got, idx[[m for m in range(n_layers) if src[m] == src[l]][0]].cpu().numpy())


def test_layer_events_mark_each_selection():
    """With per-layer events the caller waits for layer l's selection alone: a kernel on another stream
    that waits on event l reads complete rows."""
    n_layers = 4
    bs, lay, Qs, Ks, Ws = layer_inputs(n_layers, seed=95)
    side, user = torch.cuda.Stream(), torch.cuda.Stream()
    events = [torch.cuda.Event() for _ in range(n_layers)]
    idx = dsa.index_layers(lay, Qs, Ks, Ws, 24, retain_every=2, lag=1, events=events, side_stream=side)
    copies = []
    with torch.cuda.stream(user):
        for l in range(n_layers):
            user.wait_event(events[l])
            copies.append(idx[l].clone())
    user.synchronize()
    want = oracle.layer_topk(bs, 24, 2, 1)
    for l in range(n_layers):
        check_exact_sets(copies[l].cpu().numpy(), want[l], f"layer {l}")
