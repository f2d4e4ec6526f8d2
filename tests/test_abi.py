"""CPU checks of the C ABI: the library loads, exports every declared
symbol, and its host-side argument checks and workspace sizing behave as
include/dsa_index.h states (nothing here launches a kernel)."""
import ctypes
import os
import re

import pytest
import torch

import sparse_attention_indexer_04_b200 as dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(\w+)\s*\(", text, flags=re.M):
                if m.group(1) not in ("if", "for", "while", "sizeof"):
                    names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("dsa_index_scores", "dsa_index_topk", "pivot_group_index", "hisa_index", "hisa_pool_keys",
              "dsa_device_check", "dsa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(dsa.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings():
    lib = dsa.library()
    for code in range(6):
        assert lib.dsa_status_string(code).decode()
    assert lib.dsa_version() >= 100


def host_layout(q_lens, k_lens, H=4, d=32, pos=None):
    qo = torch.tensor([0] + list(torch.cumsum(torch.tensor(q_lens), 0)), dtype=torch.int32)
    ko = torch.tensor([0] + list(torch.cumsum(torch.tensor(k_lens), 0)), dtype=torch.int32)
    if pos is None:
        pos = torch.zeros(int(qo[-1]), dtype=torch.int32)
    # device arrays stand in as host tensors: nothing is dereferenced on these paths
    return dsa.Layout(qo, ko, pos, H, d, device="cpu")


def test_workspace_sizes_are_positive_and_grow():
    small = host_layout([16], [16])
    big = host_layout([4096], [4096])
    assert 0 < dsa.index_topk_workspace(small, 8) < dsa.index_topk_workspace(big, 8)
    assert dsa.index_scores_workspace(small) > 0
    assert dsa.pivot_group_index_workspace(small, 8, 4, 16, 1) > 0
    assert dsa.hisa_index_workspace(small, 8, 64, 4) > 0
    assert dsa.pivot_num_groups(host_layout([33, 16], [40, 40]), 16) == 3 + 1
    assert dsa.hisa_num_blocks(host_layout([1, 1], [300, 128]), 128) == 3 + 1


def test_hisa_workspace_holds_the_bf16_planes_of_the_pooled_keys():
    """When HISA's stages each run in one launch (at most 480 sequences, rows of at most 16,384 blocks
    and kept tokens) the workspace carries the pooled keys as three bf16 planes: 6 bytes per element."""
    L, B = 262144, 128
    lay = host_layout([2] * 4, [L] * 4, H=64, d=128, pos=torch.full((8,), L - 1, dtype=torch.int32))
    blocks = dsa.hisa_num_blocks(lay, B)
    assert blocks == 4 * L // B
    assert dsa.hisa_index_workspace(lay, 2048, B, 64) >= 3 * blocks * 128 * 2


@pytest.mark.parametrize("H,d,ok", [(4, 32, True), (64, 128, True), (3, 32, False), (4, 48, False),
                                    (128, 64, False)])
def test_unsupported_shapes_rejected(H, d, ok):
    lay = host_layout([8], [8], H=H, d=d)
    assert (dsa.index_topk_workspace(lay, 4) > 0) == ok


def call_topk(lay, k=4, Q=0x1000, K=0x2000, W=0x3000, idx=0x4000, ws=0x10000, ws_bytes=1 << 30):
    lib = dsa.library()
    return lib.dsa_index_topk(lay.ref(), ctypes.c_void_p(Q), ctypes.c_void_p(K), ctypes.c_void_p(W), k,
                              ctypes.c_void_p(idx), None, ctypes.c_void_p(ws), ctypes.c_size_t(ws_bytes), None)


def test_argument_errors_return_before_any_launch():
    lay = host_layout([8], [8])
    assert call_topk(lay, k=0) == 2                       # unsupported k
    assert call_topk(lay, k=20000) == 2
    assert call_topk(lay, Q=0x1008) == 1                  # Q not 16-byte aligned
    assert call_topk(lay, K=0x2004) == 1
    assert call_topk(lay, idx=0) == 1                     # missing output
    assert call_topk(lay, ws=0) == 3                      # missing workspace
    assert call_topk(lay, ws=0x10010) == 3                # misaligned workspace
    assert call_topk(lay, ws_bytes=16) == 3               # too small
    bad = host_layout([8], [8])
    bad.q_off_host[0] = 1
    assert call_topk(bad) == 1                            # offsets must start at 0
    bad = host_layout([8, 4], [8, 4])
    bad.k_off_host[1] = 20                                # decreasing offsets
    assert call_topk(bad) == 1
    lib = dsa.library()
    assert lib.dsa_index_topk(None, None, None, None, 4, None, None, None, 0, None) == 1
    # a row too long for the selection's shared memory (two column bitmaps) is refused up front
    assert call_topk(host_layout([1], [1_000_000]), k=2048) == 2


def test_longest_row_boundary():
    """The selection's shared memory (227 KB less 4 KB for its static part) holds the 8192-entry
    sample, a 256-entry candidate buffer and two bitmaps of ceil(n / 32) words: 774,144 columns fit,
    one more does not.  The shape check comes before the workspace check, so a row that fits
    reaches the workspace error (3) and one that does not is refused as unsupported (2)."""
    assert call_topk(host_layout([1], [774_144]), k=2048, ws_bytes=16) == 3
    assert call_topk(host_layout([1], [774_145]), k=2048, ws_bytes=16) == 2


def test_host_entry_argument_errors_need_no_gpu():
    lib = dsa.library()
    lay = host_layout([8], [8])
    P = ctypes.c_void_p
    args = lambda **kw: [lay.ref(), P(kw.get("pos", 0x800)), P(0x1000), P(0x2000), P(0x3000), kw.get("k", 4),
                         P(0x4000), P(0x10000), ctypes.c_size_t(1 << 30), P(kw.get("st", 0)), P(kw.get("si", 1)),
                         P(kw.get("so", 2))]
    assert lib.dsa_index_topk_host(*args(pos=0)) == 1          # missing positions
    assert lib.dsa_index_topk_host(*args(k=0)) == 2            # unsupported k
    assert lib.dsa_index_topk_host(*args(si=0)) == 1           # copy stream = compute stream
    assert lib.dsa_index_topk_host_workspace(lay.ref(), 4) > lib.dsa_index_topk_workspace(lay.ref(), 4)


def test_selftest_argument_errors_need_no_gpu():
    lib = dsa.library()
    P = ctypes.c_void_p
    assert lib.dsa_selftest_wait_timeout(1000, None, 256, None) == 1
    assert lib.dsa_selftest_wait_timeout(1000, P(0x10010), 256, None) == 1     # misaligned
    assert lib.dsa_selftest_wait_timeout(1000, P(0x10000), 16, None) == 1      # too small
    assert lib.dsa_selftest_wait_timeout(0, P(0x10000), 256, None) == 1        # limit out of range


def test_pivot_and_hisa_argument_errors():
    lay = host_layout([8], [8])
    lib = dsa.library()
    P = ctypes.c_void_p
    # n_cand < k, group 0, mode 2
    for k, G, C, mode in ((8, 4, 4, 0), (4, 0, 8, 0), (4, 4, 8, 2), (4, 65, 8, 0)):
        assert lib.pivot_group_index(lay.ref(), P(0x1000), P(0x2000), P(0x3000), k, G, C, mode, P(0x4000), None,
                                     P(0x10000), ctypes.c_size_t(1 << 30), None) == 2
    for k, B, keep in ((4, 100, 4), (4, 128, 0), (0, 128, 4)):
        assert lib.hisa_index(lay.ref(), P(0x1000), P(0x2000), P(0x3000), P(0x5000), k, B, keep, P(0x4000), None,
                              P(0x10000), ctypes.c_size_t(1 << 30), None) == 2


def test_layer_schedule_host_function_matches_oracle():
    """dsa_index_layers_source (host-only) against the oracle's stepwise reading of IndexCache and MLI."""
    import oracle
    for n in range(1, 12):
        for r in (1, 2, 3, 4, 8):
            for lag in (0, 1):
                want = oracle.layer_sources(n, r, lag)
                got = [dsa.index_layers_source(l, r, lag) for l in range(n)]
                assert got == want, (n, r, lag)
    assert dsa.index_layers_source(-1, 2, 0) == -1
    assert dsa.index_layers_source(3, 0, 0) == -1
    assert dsa.index_layers_source(3, 2, 2) == -1


def test_checked_build_exports_the_same_entry_points():
    """libdsaidx_checked.so (the build whose kernels verify their device-side indices) exports every
    declared entry point too."""
    path = os.path.join(ROOT, "sparse_attention_indexer_04_b200", "libdsaidx_checked.so")
    lib = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(lib, name), name
