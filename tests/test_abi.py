"""The C-ABI library without a GPU: it builds, loads, exports every symbol the header
declares, and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest
import torch

import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import _abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lsa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load()


def test_header_declares_the_six_calls():
    names = declared_functions()
    for call in ("lsa_index_score", "lsa_select_union", "lsa_compact", "lsa_topk",
                 "lsa_gather_cold", "lsa_vote_labels"):
        assert call in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(_abi.SIGNATURES) == set(declared_functions())


def test_status_strings_and_version(lib):
    assert lib.lsa_abi_version() == 1
    for code in range(8):
        assert lib.lsa_status_string(code)
    assert lsa.status_string(3) == "list longer than its capacity"


def test_host_side_argument_errors(lib):
    # Each of these returns before any CUDA call.
    assert lib.lsa_select_union(-1, 4, None, None, None, None) == lsa.LSA_ERR_INVALID_ARG
    assert lib.lsa_select_union(2, 4, None, None, None, None) == lsa.LSA_ERR_INVALID_ARG
    assert lib.lsa_select_union(0, 4, None, None, None, None) == lsa.LSA_OK
    assert lib.lsa_compact(1, 64, None, 8, None, None, None, None) == lsa.LSA_ERR_INVALID_ARG
    assert lib.lsa_gather_cold(1, 4, 24, 16, 16, 16, 4, 16, None, None) == lsa.LSA_ERR_INVALID_ARG
    assert b"multiple of 16" in lib.lsa_last_error()
    assert lib.lsa_topk(1, 0, 10, 4, 16, 4, 16, 16, 16, None, None, 0, None) == lsa.LSA_ERR_INVALID_ARG
    assert lib.lsa_vote_labels(2, 2, 8, 16, ctypes.c_float(1.5), 3, 16, None, None,
                               ctypes.c_float(2.0), None, None, 0, None) == lsa.LSA_ERR_INVALID_ARG
    args = [1, 1, 128, 64, 16, 8, 64]
    rc = lib.lsa_index_score(*args, 7, None, None, None, None, None, 0, None, None, 0,
                             None, None, None, None, None, None, None, None, None, 0, None)
    assert rc == lsa.LSA_ERR_UNSUPPORTED
    rc = lib.lsa_index_score(*args, 0, 256, 256, 256, 256, 256, 2, 256, None, 0,
                             None, None, None, None, 256, None, None, None, None, 0, None)
    assert rc == lsa.LSA_ERR_INVALID_ARG            # e4m3 keys without a scale
    rc = lib.lsa_index_score(*args, 0, 256, 256, 256, 256, 256, 0, 256, None, 0,
                             None, None, None, None, 256, None, None, None, None, 0, None)
    assert rc == lsa.LSA_ERR_NOMEM                  # no workspace
    # size limits: sequence x layer pairs, layers per call, training positions
    rc = lib.lsa_index_score(30000, 3, 128, 64, 16, 8, 64, 0, 256, 256, 256, 256, 256, 0, 256, None, -1,
                             None, None, None, None, 256, None, None, None, None, 0, None)
    assert rc == lsa.LSA_ERR_UNSUPPORTED and b"65535" in lib.lsa_last_error()
    rc = lib.lsa_index_project(1, 70000, 64, 16, 8, 64, 0, 256, 256, 256, 256, -1, 256, 256, None, 0, None)
    assert rc == lsa.LSA_ERR_UNSUPPORTED and b"65535" in lib.lsa_last_error()
    rc = lib.lsa_index_train_step(4097, 256, 64, 16, 128, 64, 1, 256, 256, 256, 256, ctypes.c_float(0.0), 1, 256,
                                  None, 256, ctypes.c_float(2.0), 256, 256, 256, None, 256, 256, 256, None, None,
                                  None, 0, None)
    assert rc == lsa.LSA_ERR_UNSUPPORTED and b"at most 4096" in lib.lsa_last_error()
    upd = lib.lsa_hot_pool_update
    assert upd(1, 64, 8, 1152, 0, 256, 256, 256, 256, None, None, 256, 1 << 20, None) == lsa.LSA_ERR_INVALID_ARG
    assert b"trigger" in lib.lsa_last_error()
    assert upd(1, 64, 0, 1152, 1, 256, 256, 256, 256, None, None, 256, 1 << 20, None) == lsa.LSA_ERR_INVALID_ARG
    assert upd(1, 64, 8, 24, 1, 256, 256, 256, 256, None, None, 256, 1 << 20, None) == lsa.LSA_ERR_INVALID_ARG
    assert upd(1, 64, 8, 1152, 1, None, 256, 256, 256, None, None, 256, 1 << 20, None) == lsa.LSA_ERR_INVALID_ARG
    assert upd(1, 64, 8, 1152, 1, 256, 256, 256, 264, None, None, 256, 1 << 20, None) == lsa.LSA_ERR_INVALID_ARG
    assert upd(1, 64, 8, 1152, 1, 256, 256, 256, 256, None, None, 256, 16, None) == lsa.LSA_ERR_NOMEM
    assert lib.lsa_hot_pool_reset(1, 64, 8, None, None) == lsa.LSA_ERR_INVALID_ARG


def test_binding_refuses_strided_views(lib):
    # marshalling only, but a transposed view would be read as dense: refused before the call
    bits = torch.zeros(2, 4, dtype=torch.int32)
    with pytest.raises(ValueError, match="not contiguous"):
        lsa.lsa_compact(4, 64, bits.t(), 8, torch.zeros(4, 8, dtype=torch.int32), torch.zeros(4, dtype=torch.int32),
                        stream=0)
    with pytest.raises(lsa.LsaError):       # a dense tensor reaches the library (which refuses the null list)
        lsa.lsa_compact(4, 64, bits.reshape(4, 2), 8, None, torch.zeros(4, dtype=torch.int32), stream=0)


def test_hot_pool_layout():
    B, N, slots = 3, 1000, 40
    off = lsa.lsa_hot_pool_layout(B, N, slots)
    assert off[0] == 0 and all(o % 256 == 0 for o in off)
    assert off[1] >= B * N * 4 and off[2] >= off[1] + B * slots * 4 and off[3] >= off[2] + B * slots * 4
    assert lsa.lsa_hot_pool_state_bytes(B, N, slots) >= off[3] + B * ((N + 31) // 32) * 4
    assert lsa.lsa_hot_pool_workspace_bytes(B, N, slots) > 0


def test_workspace_queries(lib):
    n = lib.lsa_index_score_workspace_bytes(32, 3, 262144, 4096, 512, 64, 128, 1, 2)
    assert 0 < n < 64 << 20
    assert lib.lsa_topk_workspace_bytes(32, 262144) >= 32 * 262144 * 4
    assert lib.lsa_vote_labels_workspace_bytes(24, 64, 131072) >= 24 * 64 * 4096 * 4


def test_selection_and_keyed_topk_argument_errors(lib):
    """The fused selection and the keyed top-k refuse bad arguments on the host (fake,
    aligned device addresses; every case returns before a launch)."""
    A = 256                                   # an aligned non-null address, never dereferenced
    B, L, N = 2, 3, 4096
    ws_need = lib.lsa_select_fetch_workspace_bytes(B, N)
    Nw = (N + 31) // 32
    # the per-chunk counts, the union's warp bases and a copy of the union words fit
    assert ws_need >= B * Nw * 4 + B * ((Nw + 255) // 256) * 9 * 4
    sf = lib.lsa_select_fetch
    args = lambda **kw: [kw.get("B", B), kw.get("L", L), N, A, None, None, N, A, A, A, A,
                         kw.get("logit", None), kw.get("key_U", None), None, kw.get("ws", A),
                         kw.get("wsb", ws_need), None]
    assert sf(*args(L=9)) == lsa.LSA_ERR_UNSUPPORTED and b"1 to 8" in lib.lsa_last_error()
    assert sf(*args(B=-1)) == lsa.LSA_ERR_INVALID_ARG
    assert sf(*args(key_U=A)) == lsa.LSA_ERR_INVALID_ARG and b"needs the logits" in lib.lsa_last_error()
    assert sf(*args(logit=A, key_U=A + 4)) == lsa.LSA_ERR_INVALID_ARG      # key_U not 16-byte aligned
    assert sf(*args(wsb=ws_need - 1)) == lsa.LSA_ERR_NOMEM
    assert sf(*args(ws=A + 16)) == lsa.LSA_ERR_NOMEM                       # workspace not 256-byte aligned
    assert sf(*args(B=0)) == lsa.LSA_OK
    tk = lib.lsa_topk_keyed
    assert tk(-1, 8, A, N, A, A, A, A, None) == lsa.LSA_ERR_INVALID_ARG
    assert tk(B, 8, A, N, None, A, A, A, None) == lsa.LSA_ERR_INVALID_ARG   # no counts
    assert tk(B, 8, A, N, A, A, None, A, None) == lsa.LSA_ERR_INVALID_ARG   # k > 0 without an output
    assert tk(B, 8, A, N, A, A + 2, A, A, None) == lsa.LSA_ERR_INVALID_ARG  # keys not 4-byte aligned
    assert tk(0, 8, A, N, A, A, A, A, None) == lsa.LSA_OK
