"""Python binding of libdsaidx, the B200 DSA lightning-indexer library.

Argument marshalling only: every step of the indexer runs in the library's
CUDA kernels.  Tensors are torch CUDA tensors (PyTorch supplies device
memory and the current stream); the library itself allocates nothing, so
outputs and workspaces are allocated here with torch and handed over as raw
pointers.  There is no CPU fallback: importing this package fails loudly
when the compiled library is missing.

Entry points mirror include/dsa_index.h:
  index_scores, index_topk, index_topk_host, index_layers, pivot_group_index,
  pivot_refine_candidates, hisa_pool_keys, hisa_index, device_check, plus the
  *_workspace size queries.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# DSA_LIBRARY=checked loads the build whose kernels verify their device-side indices; every entry
# point then also reads the workspace status word after its work (synchronising) and raises on a
# recorded error.
CHECKED = os.environ.get("DSA_LIBRARY", "") == "checked"
LIB_PATH = os.path.join(_HERE, "libdsaidx_checked.so" if CHECKED else "libdsaidx.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python sparse_attention_indexer_04_b200/build.py` "
                      "(or __graft_entry__.build()); there is no fallback path")
_lib = ctypes.CDLL(LIB_PATH)

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "workspace", 4: "CUDA error",
          5: "device check"}
REUSE, REFINE = 0, 1


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.dsa_status_string(status).decode()} (status {status})")


class _Batch(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("num_queries", ctypes.c_int32), ("num_keys", ctypes.c_int32),
                ("q_offsets", ctypes.c_void_p), ("k_offsets", ctypes.c_void_p), ("q_pos", ctypes.c_void_p),
                ("q_offsets_host", ctypes.c_void_p), ("k_offsets_host", ctypes.c_void_p)]


_P = ctypes.c_void_p
_B = ctypes.POINTER(_Batch)
_I32, _I64, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("dsa_status_string", ctypes.c_char_p, ctypes.c_int)
_sig("dsa_version", _I32)
_sig("dsa_index_scores_workspace", _SZ, _B)
_sig("dsa_index_scores", ctypes.c_int, _B, _P, _P, _P, _P, _I64, _P, _SZ, _P)
_sig("dsa_index_topk_workspace", _SZ, _B, _I32)
_sig("dsa_index_topk", ctypes.c_int, _B, _P, _P, _P, _I32, _P, _P, _P, _SZ, _P)
_sig("dsa_index_topk_host_workspace", _SZ, _B, _I32)
_sig("dsa_index_topk_host", ctypes.c_int, _B, _P, _P, _P, _P, _I32, _P, _P, _SZ, _P, _P, _P)
_sig("pivot_num_groups", _I32, _B, _I32)
_sig("pivot_group_index_workspace", _SZ, _B, _I32, _I32, _I32, _I32)
_sig("pivot_group_index", ctypes.c_int, _B, _P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _SZ, _P)
_sig("pivot_refine_candidates_workspace", _SZ, _B, _I32, _I32, _I32)
_sig("pivot_refine_candidates", ctypes.c_int, _B, _P, _P, _P, _I32, _I32, _I32, _P, _P, _P, _SZ, _P)
_sig("hisa_num_blocks", _I64, _B, _I32)
_sig("hisa_pool_keys", ctypes.c_int, _B, _P, _I32, _P, _P)
_sig("hisa_index_workspace", _SZ, _B, _I32, _I32, _I32)
_sig("hisa_index", ctypes.c_int, _B, _P, _P, _P, _P, _I32, _I32, _I32, _P, _P, _P, _SZ, _P)
_sig("dsa_device_check", ctypes.c_int, _P, _P, ctypes.POINTER(ctypes.c_uint32))
_sig("dsa_selftest_wait_timeout", ctypes.c_int, ctypes.c_uint32, _P, _SZ, _P)
_sig("dsa_index_topk_static_capacity", _SZ)
_sig("dsa_index_topk_static", ctypes.c_int, _B, _P, _P, _P, _I32, _P, _P, _P)
_sig("dsa_index_layers_source", _I32, _I32, _I32, _I32)
_sig("dsa_index_layers_workspace", _SZ, _B, _I32)
_sig("dsa_index_layers", ctypes.c_int, _B, _I32, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P), _I32,
     _I32, _I32, ctypes.POINTER(_P), ctypes.POINTER(_P), _P, _SZ, _P, _P)
_sig("dsa_profile_enable", None, _I32)
_sig("dsa_launch_count", ctypes.c_uint64)
_sig("dsa_profile_kind_name", ctypes.c_char_p, _I32)
_sig("dsa_profile_read", _I32, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int32), _I32)


def library():
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise DsaError(status, where)


ERR_BAD_INDEX = 4   # status-word code of the checked build: a device-side index outside its buffer


def _after(ws, where: str, stream=None):
    """Checked build only: wait for the call's work and raise if a kernel recorded an index error in
    the workspace status word (other codes are left for device_check)."""
    if not CHECKED:
        return
    torch.cuda.synchronize()   # every stream the call used
    code, detail = (int(x) for x in ws[:8].view(torch.int32).cpu())
    if code == ERR_BAD_INDEX:
        raise DsaError(5, f"{where}: device index check failed at site {detail}")


class Layout:
    """Sequence layout of a batch: offsets and positions on the device plus host copies.

    q_offsets / k_offsets: [B+1] row offsets of each sequence's queries / keys;
    q_pos: [n_q] sequence-local position of each query.
    """

    def __init__(self, q_offsets, k_offsets, q_pos, num_heads: int, head_dim: int, device="cuda"):
        self.q_off_host = torch.as_tensor(q_offsets, dtype=torch.int32).cpu().contiguous()
        self.k_off_host = torch.as_tensor(k_offsets, dtype=torch.int32).cpu().contiguous()
        self.q_off = self.q_off_host.to(device)
        self.k_off = self.k_off_host.to(device)
        self.q_pos = torch.as_tensor(q_pos, dtype=torch.int32).to(device).contiguous()
        self.num_heads, self.head_dim = int(num_heads), int(head_dim)
        self.device = torch.device(device)
        self.c = _Batch(int(self.q_off_host.numel() - 1), self.num_heads, self.head_dim,
                        int(self.q_off_host[-1]), int(self.k_off_host[-1]),
                        self.q_off.data_ptr(), self.k_off.data_ptr(),
                        self.q_pos.data_ptr() if self.q_pos.numel() else None,
                        self.q_off_host.data_ptr(), self.k_off_host.data_ptr())

    @classmethod
    def from_batch(cls, b, device="cuda"):
        return cls(b.q_offsets, b.k_offsets, b.q_pos, b.H, b.d, device)

    @property
    def num_queries(self):
        return self.c.num_queries

    @property
    def max_keys(self):
        ko = self.k_off_host
        return int((ko[1:] - ko[:-1]).max()) if ko.numel() > 1 else 0

    def ref(self):
        return ctypes.byref(self.c)


def _workspace(nbytes: int, device, ws=None):
    if ws is not None:
        return ws
    # 256-byte aligned: torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _bytes(ws):
    return ctypes.c_size_t(ws.numel() * ws.element_size())


# ------------------------------------------------------------------- dense

def index_scores_workspace(layout: Layout) -> int:
    return int(_lib.dsa_index_scores_workspace(layout.ref()))


def index_scores(layout: Layout, Q, K, W, S=None, ws=None, stream=None):
    """Dense indexer scores: S [n_q, ld] fp32, -inf where the key is not eligible."""
    if S is None:
        S = torch.empty(layout.num_queries, max(layout.max_keys, 1), dtype=torch.float32, device=layout.device)
    ws = _workspace(index_scores_workspace(layout), layout.device, ws)
    _check(_lib.dsa_index_scores(layout.ref(), _ptr(Q), _ptr(K), _ptr(W), _ptr(S), S.stride(0), _ptr(ws),
                                 _bytes(ws), _stream(stream)), "dsa_index_scores")
    _after(ws, "dsa_index_scores", stream)
    return S


def index_topk_workspace(layout: Layout, k: int) -> int:
    return int(_lib.dsa_index_topk_workspace(layout.ref(), k))


def index_topk(layout: Layout, Q, K, W, k: int, idx=None, scores=None, want_scores=False, ws=None, stream=None):
    """Dense indexer top-k: idx [n_q, k] int32 (ascending, -1 padded), optional scores [n_q, k]."""
    if idx is None:
        idx = torch.empty(layout.num_queries, k, dtype=torch.int32, device=layout.device)
    if want_scores and scores is None:
        scores = torch.empty(layout.num_queries, k, dtype=torch.float32, device=layout.device)
    ws = _workspace(index_topk_workspace(layout, k), layout.device, ws)
    _check(_lib.dsa_index_topk(layout.ref(), _ptr(Q), _ptr(K), _ptr(W), k, _ptr(idx), _ptr(scores), _ptr(ws),
                               _bytes(ws), _stream(stream)), "dsa_index_topk")
    _after(ws, "dsa_index_topk", stream)
    return (idx, scores) if want_scores else idx


def index_layers_source(layer: int, retain_every: int, lag: int) -> int:
    """The layer whose indexer run gives `layer` its selection (-1 for invalid arguments)."""
    return int(_lib.dsa_index_layers_source(layer, retain_every, lag))


def index_layers(layout: Layout, Qs, Ks, Ws, k: int, retain_every: int = 1, lag: int = 0, idx=None, events=None,
                 ws=None, stream=None, side_stream=None):
    """Selections of len(Qs) layers (dsa_index_layers): idx[l] [n_q, k] int32 for layer l.  `events`: optional
    torch.cuda.Event per layer, recorded once idx[l] is complete (then `stream` is not made to wait)."""
    n = len(Qs)
    if not (len(Ks) == len(Ws) == n):
        raise ValueError("one Q, K and W per layer")
    if idx is None:
        idx = [torch.empty(layout.num_queries, k, dtype=torch.int32, device=layout.device) for _ in range(n)]
    if side_stream is None:
        raise ValueError("index_layers needs a side stream distinct from the compute stream")
    arr = lambda ts: (_P * n)(*[t.data_ptr() for t in ts])
    ev = None
    if events is not None:
        for e in events:
            e.record(stream if stream is not None else torch.cuda.current_stream())   # creates the event
        ev = (_P * n)(*[e.cuda_event for e in events])
    ws = _workspace(int(_lib.dsa_index_layers_workspace(layout.ref(), k)), layout.device, ws)
    _check(_lib.dsa_index_layers(layout.ref(), n, arr(Qs), arr(Ks), arr(Ws), k, retain_every, lag, arr(idx), ev,
                                 _ptr(ws), _bytes(ws), _stream(stream), _stream(side_stream)), "dsa_index_layers")
    _after(ws, "dsa_index_layers", stream)
    return idx


def index_topk_host_workspace(layout: Layout, k: int) -> int:
    return int(_lib.dsa_index_topk_host_workspace(layout.ref(), k))


def index_topk_host(layout: Layout, q_pos, Q, K, W, k: int, idx, ws, stream=None, in_stream=None, out_stream=None):
    """dsa_index_topk on HOST tensors (pinned for overlap): Q, K, W, q_pos (CPU) in, idx [n_q, k] (CPU,
    int32) out.  The copies run on in_stream / out_stream (torch.cuda.Stream) overlapped with the
    work on `stream`; idx is complete once `stream` has passed the call."""
    for t in (q_pos, Q, K, W, idx):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("index_topk_host takes contiguous host tensors")
    if in_stream is None or out_stream is None:
        raise ValueError("index_topk_host needs copy streams distinct from the compute stream")
    _check(_lib.dsa_index_topk_host(layout.ref(), _ptr(q_pos), _ptr(Q), _ptr(K), _ptr(W), k, _ptr(idx), _ptr(ws),
                                    _bytes(ws), _stream(stream), _stream(in_stream), _stream(out_stream)),
           "dsa_index_topk_host")
    _after(ws, "dsa_index_topk_host", stream)
    return idx


def index_topk_static(layout: Layout, Q, K, W, k: int, idx=None, scores=None, want_scores=False, stream=None):
    """dsa_index_topk with the library's built-in device scratch instead of a workspace (allocates nothing
    in the library; for callers that cannot allocate).  Calls on one device must not overlap on the GPU."""
    if idx is None:
        idx = torch.empty(layout.num_queries, k, dtype=torch.int32, device=layout.device)
    if want_scores and scores is None:
        scores = torch.empty(layout.num_queries, k, dtype=torch.float32, device=layout.device)
    _check(_lib.dsa_index_topk_static(layout.ref(), _ptr(Q), _ptr(K), _ptr(W), k, _ptr(idx), _ptr(scores),
                                      _stream(stream)), "dsa_index_topk_static")
    return (idx, scores) if want_scores else idx


def index_topk_static_capacity() -> int:
    return int(_lib.dsa_index_topk_static_capacity())


# ------------------------------------------------------------------- PIVOT

def pivot_num_groups(layout: Layout, group: int) -> int:
    return int(_lib.pivot_num_groups(layout.ref(), group))


def pivot_group_index_workspace(layout: Layout, k: int, group: int, n_cand: int, mode: int) -> int:
    return int(_lib.pivot_group_index_workspace(layout.ref(), k, group, n_cand, mode))


def pivot_group_index(layout: Layout, Q, K, W, k: int, group: int, n_cand: int, mode: int, idx=None, cand=None,
                      want_cand=False, ws=None, stream=None):
    """PIVOT Reuse (mode 0) / Refine (mode 1): idx [n_q, k]; optional cand [n_groups, n_cand]."""
    if idx is None:
        idx = torch.empty(layout.num_queries, k, dtype=torch.int32, device=layout.device)
    if want_cand and cand is None:
        cand = torch.empty(max(pivot_num_groups(layout, group), 0), n_cand, dtype=torch.int32, device=layout.device)
    ws = _workspace(pivot_group_index_workspace(layout, k, group, n_cand, mode), layout.device, ws)
    _check(_lib.pivot_group_index(layout.ref(), _ptr(Q), _ptr(K), _ptr(W), k, group, n_cand, mode, _ptr(idx),
                                  _ptr(cand), _ptr(ws), _bytes(ws), _stream(stream)), "pivot_group_index")
    _after(ws, "pivot_group_index", stream)
    return (idx, cand) if want_cand else idx


def pivot_refine_candidates_workspace(layout: Layout, k: int, group: int, n_cand: int) -> int:
    return int(_lib.pivot_refine_candidates_workspace(layout.ref(), k, group, n_cand))


def pivot_refine_candidates(layout: Layout, Q, K, W, k: int, group: int, cand, idx=None, ws=None, stream=None):
    """Refine on supplied candidates: cand [n_groups, n_cand] int32 (ascending, -1 padded) -> idx [n_q, k]."""
    n_cand = int(cand.shape[1])
    if idx is None:
        idx = torch.empty(layout.num_queries, k, dtype=torch.int32, device=layout.device)
    ws = _workspace(pivot_refine_candidates_workspace(layout, k, group, n_cand), layout.device, ws)
    _check(_lib.pivot_refine_candidates(layout.ref(), _ptr(Q), _ptr(K), _ptr(W), k, group, n_cand, _ptr(cand),
                                        _ptr(idx), _ptr(ws), _bytes(ws), _stream(stream)), "pivot_refine_candidates")
    _after(ws, "pivot_refine_candidates", stream)
    return idx


# -------------------------------------------------------------------- HISA

def hisa_num_blocks(layout: Layout, block: int) -> int:
    return int(_lib.hisa_num_blocks(layout.ref(), block))


def hisa_pool_keys(layout: Layout, K, block: int, pooled=None, stream=None):
    """Mean-pooled block keys [n_blocks, d] fp32."""
    if pooled is None:
        pooled = torch.empty(max(hisa_num_blocks(layout, block), 0), layout.head_dim, dtype=torch.float32,
                             device=layout.device)
    _check(_lib.hisa_pool_keys(layout.ref(), _ptr(K), block, _ptr(pooled), _stream(stream)), "hisa_pool_keys")
    return pooled


def hisa_index_workspace(layout: Layout, k: int, block: int, keep: int) -> int:
    return int(_lib.hisa_index_workspace(layout.ref(), k, block, keep))


def hisa_index(layout: Layout, Q, K, W, pooled, k: int, block: int, keep: int, idx=None, kept=None,
               want_kept=False, ws=None, stream=None):
    """HISA top-k: idx [n_q, k]; optional kept [n_q, keep+2] block lists."""
    if idx is None:
        idx = torch.empty(layout.num_queries, k, dtype=torch.int32, device=layout.device)
    if want_kept and kept is None:
        kept = torch.empty(layout.num_queries, keep + 2, dtype=torch.int32, device=layout.device)
    ws = _workspace(hisa_index_workspace(layout, k, block, keep), layout.device, ws)
    _check(_lib.hisa_index(layout.ref(), _ptr(Q), _ptr(K), _ptr(W), _ptr(pooled), k, block, keep, _ptr(idx),
                           _ptr(kept), _ptr(ws), _bytes(ws), _stream(stream)), "hisa_index")
    _after(ws, "hisa_index", stream)
    return (idx, kept) if want_kept else idx


def launch_count() -> int:
    """Kernels this library has launched since it was loaded."""
    return int(_lib.dsa_launch_count())


def profile_enable(on: bool = True):
    """Bracket every later launch with CUDA events on its own stream (see profile_read)."""
    _lib.dsa_profile_enable(1 if on else 0)


def profile_read():
    """{kernel kind: (total ms, launches)} since the last read; synchronises the recorded events."""
    cap = 32
    ms = (ctypes.c_float * cap)()
    n = (ctypes.c_int32 * cap)()
    kinds = _lib.dsa_profile_read(ms, n, cap)
    if kinds < 0:
        raise DsaError(4, "dsa_profile_read")
    return {_lib.dsa_profile_kind_name(i).decode(): (float(ms[i]), int(n[i])) for i in range(kinds) if n[i]}


def selftest_wait_timeout(limit_us: int, ws, stream=None):
    """Launch the bounded-wait self-test: a wait nothing completes runs out after limit_us and records
    code 1 in ws's status word (read it with device_check)."""
    _check(_lib.dsa_selftest_wait_timeout(limit_us, _ptr(ws), _bytes(ws), _stream(stream)),
           "dsa_selftest_wait_timeout")


def device_check(ws, stream=None) -> int:
    """Status word recorded by kernels in a workspace (0 = none); synchronises the stream."""
    detail = ctypes.c_uint32(0)
    st = _lib.dsa_device_check(_ptr(ws), _stream(stream), ctypes.byref(detail))
    if st not in (0, 5):
        raise DsaError(st, "dsa_device_check")
    return int(detail.value) if st == 5 else 0
