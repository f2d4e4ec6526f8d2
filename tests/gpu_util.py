"""Helpers shared by the GPU parity tests: move a workloads.Batch to the
device and call the library through its C ABI binding."""
import numpy as np
import torch

import sparse_attention_indexer_04_b200 as dsa


class Dev:
    def __init__(self, b, device="cuda:0"):
        self.b = b
        self.dev = torch.device(device)
        self.lay = dsa.Layout.from_batch(b, self.dev)
        self.Q = b.Q.to(self.dev)
        self.K = b.K.to(self.dev)
        self.W = b.W.to(self.dev)

    def topk(self, k, want_scores=False):
        out = dsa.index_topk(self.lay, self.Q, self.K, self.W, k, want_scores=want_scores)
        torch.cuda.synchronize()
        if want_scores:
            return out[0].cpu().numpy(), out[1].cpu().numpy()
        return out.cpu().numpy()

    def scores(self):
        S = dsa.index_scores(self.lay, self.Q, self.K, self.W)
        torch.cuda.synchronize()
        return S.cpu().numpy()

    def pivot(self, k, G, C, mode):
        idx, cand = dsa.pivot_group_index(self.lay, self.Q, self.K, self.W, k, G, C, mode, want_cand=True)
        torch.cuda.synchronize()
        return idx.cpu().numpy(), cand.cpu().numpy()

    def pivot_idx(self, k, G, C, mode):
        """Indices only (no candidate list asked for: Reuse then selects the group lists from the proxy
        rows directly)."""
        idx = dsa.pivot_group_index(self.lay, self.Q, self.K, self.W, k, G, C, mode)
        torch.cuda.synchronize()
        return idx.cpu().numpy()

    def hisa(self, k, B, keep):
        pooled = dsa.hisa_pool_keys(self.lay, self.K, B)
        idx, kept = dsa.hisa_index(self.lay, self.Q, self.K, self.W, pooled, k, B, keep, want_kept=True)
        torch.cuda.synchronize()
        return idx.cpu().numpy(), kept.cpu().numpy(), pooled.cpu().numpy()


def ascending_packed(rows):
    """Library rows: valid indices ascending, then -1."""
    for r in rows:
        v = r[r >= 0]
        n = v.size
        assert np.all(r[n:] == -1), "padding must follow the valid entries"
        assert np.all(np.diff(v) > 0), "valid entries must be strictly ascending"
