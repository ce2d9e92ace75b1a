"""Parity of the selection calls (union, compact, top-k, gather) with the oracle."""
import numpy as np
import pytest
import torch

import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import build
from oracle import lsa_oracle as O

import lsa_cases as C

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    lsa.lib()


def bits_tensor(mark: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(O.pack_bits(mark).view(np.int32).copy()).cuda()


def test_union_incremental_exact():
    g = np.random.default_rng(0)
    B, N = 5, 3000
    marks = [g.random((B, N)) < p for p in (0.1, 0.3, 0.05)]
    Nw = (N + 31) // 32
    U = torch.zeros(B, Nw, dtype=torch.int32, device="cuda")
    news = []
    for m in marks:
        nw = torch.zeros(B, Nw, dtype=torch.int32, device="cuda")
        lsa.lsa_select_union(B, Nw, bits_tensor(m), U, nw)
        news.append(nw)
    torch.cuda.synchronize()
    for b in range(B):
        Ue, newe = O.or_union([m[b] for m in marks])
        assert np.array_equal(C.unpack(U[b], N), Ue)
        for l in range(3):
            assert np.array_equal(C.unpack(news[l][b], N), newe[l])


@pytest.mark.parametrize("N,p", [(1, 1.0), (33, 0.5), (70000, 0.2), (262144, 0.01), (5000, 0.0)])
def test_compact_exact(N, p):
    g = np.random.default_rng(N)
    B = 3
    m = g.random((B, N)) < p
    cap = N
    idx = torch.full((B, max(cap, 1)), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.lsa_compact(B, N, bits_tensor(m), cap, idx, cnt, st)
    torch.cuda.synchronize()
    assert int(st) == 0
    for b in range(B):
        e = O.compact(m[b])
        assert int(cnt[b]) == len(e)
        assert np.array_equal(idx[b, : len(e)].cpu().numpy(), e)


@pytest.mark.parametrize("N", [40, 100])
def test_compact_more_sequences_than_one_launch(N):
    """70,000 sequences: more than one launch's 65,535 (the sequence is the grid's y
    index), with word rows that are and are not 16-byte multiples."""
    g = np.random.default_rng(N + 7)
    B, cap = 70000, N
    m = g.random((B, N)) < 0.3
    idx = torch.full((B, cap), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.lsa_compact(B, N, bits_tensor(m), cap, idx, cnt, st)
    torch.cuda.synchronize()
    assert int(st) == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(B):
        e = O.compact(m[b])
        assert cnt[b] == len(e), b
        assert np.array_equal(idx[b, : len(e)], e), b
        assert (idx[b, len(e):] == -7).all(), b


def test_compact_capacity_overflow_sets_status():
    g = np.random.default_rng(1)
    B, N, cap = 2, 5000, 100
    m = g.random((B, N)) < 0.3
    idx = torch.full((B, cap), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.lsa_compact(B, N, bits_tensor(m), cap, idx, cnt, st)
    torch.cuda.synchronize()
    assert int(st) == lsa.LSA_ERR_CAPACITY
    for b in range(B):
        e = O.compact(m[b])
        assert int(cnt[b]) == len(e)
        assert np.array_equal(idx[b].cpu().numpy(), e[:cap])


def run_topk(idx_list, logits, k, N):
    L, B = logits.shape[0], len(idx_list)
    cap = max(1, max(len(x) for x in idx_list))
    idx = torch.full((B, cap), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    for b, x in enumerate(idx_list):
        idx[b, : len(x)] = torch.from_numpy(np.asarray(x, dtype=np.int32))
        cnt[b] = len(x)
    topk = torch.full((B, max(k, 1)), -9, dtype=torch.int32, device="cuda")
    tc = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_topk_workspace_bytes(B, cap))
    lsa.lsa_topk(B, L, N, k, idx, cap, cnt, torch.from_numpy(logits).cuda(), topk, tc, ws)
    torch.cuda.synchronize()
    return topk.cpu().numpy(), tc.cpu().numpy()


@pytest.mark.parametrize("k", [0, 1, 7, 64, 512])
def test_topk_exact_with_ties(k):
    g = np.random.default_rng(k)
    L, B, N = 3, 4, 6000
    logits = np.round(g.standard_normal((L, B, N)) * 4, 1).astype(np.float32)   # many ties
    idx_list = [np.sort(g.choice(N, size=int(n), replace=False)) for n in (0, 5, 900, 5999)]
    topk, tc = run_topk(idx_list, logits, k, N)
    for b in range(B):
        key = logits[:, b, :].astype(np.float64).max(axis=0)
        e = O.topk_in_fetched(idx_list[b], key, k)
        assert tc[b] == len(e)
        assert np.array_equal(topk[b, : len(e)], e)
        assert np.all(topk[b, len(e): k] == -1)


def check_topk(idx_list, logits, k, topk, tc):
    for b in range(len(idx_list)):
        key = logits[:, b, :].astype(np.float64).max(axis=0)
        e = O.topk_in_fetched(idx_list[b], key, k)
        assert tc[b] == len(e)
        assert np.array_equal(topk[b, : len(e)], e), b
        assert np.all(topk[b, len(e): k] == -1)


def test_topk_many_sequences_keys_beyond_shared_memory():
    """150 sequences (one CTA each on a 148-SM part); 60,000 candidates exceed one CTA's
    shared-memory key slice, so those keys live in the workspace."""
    g = np.random.default_rng(21)
    L, B, N, k = 2, 150, 60000, 2048
    logits = np.round(g.standard_normal((L, B, N)) * 3, 1).astype(np.float32)   # ties at the k-th key
    sizes = [N if b % 3 == 0 else (50000 if b % 3 == 1 else int(g.integers(0, 5000))) for b in range(B)]
    idx_list = [np.arange(N) if n == N else np.sort(g.choice(N, size=n, replace=False)) for n in sizes]
    topk, tc = run_topk(idx_list, logits, k, N)
    check_topk(idx_list, logits, k, topk, tc)


def test_topk_long_sequences_cluster_slices():
    """Two sequences split over a cluster of CTAs: 300,000 candidates (keys in shared
    memory) and 450,000 (slices beyond shared memory)."""
    g = np.random.default_rng(22)
    L, B, N, k = 3, 2, 500000, 2048
    logits = np.round(g.standard_normal((L, B, N)) * 4, 2).astype(np.float32)
    idx_list = [np.sort(g.choice(N, size=300000, replace=False)), np.sort(g.choice(N, size=450000, replace=False))]
    topk, tc = run_topk(idx_list, logits, k, N)
    check_topk(idx_list, logits, k, topk, tc)


def test_topk_negative_keys_and_all_equal():
    L, B, N = 1, 2, 3000
    logits = np.full((L, B, N), -2.5, dtype=np.float32)
    logits[0, 1] = -np.arange(N, dtype=np.float32)   # strictly decreasing
    idx = [np.arange(N), np.arange(0, N, 3)]
    topk, tc = run_topk(idx, logits, 100, N)
    assert np.array_equal(topk[0, :100], np.arange(100))            # all ties -> lowest indices
    assert np.array_equal(topk[1, :100], np.arange(0, 300, 3))


def test_gather_bytes_exact_and_range_status():
    g = np.random.default_rng(2)
    B, N, R = 3, 4000, 1152
    cold = torch.from_numpy(g.integers(0, 256, size=(B, N, R), dtype=np.uint8)).pin_memory()
    lists = [np.sort(g.choice(N, size=n, replace=False)) for n in (0, 17, 2500)]
    cap = 2600
    idx = torch.zeros(B, cap, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    for b, x in enumerate(lists):
        idx[b, : len(x)] = torch.from_numpy(x.astype(np.int32))
        cnt[b] = len(x)
    hot = torch.zeros(B, cap, R, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        lsa.lsa_gather_cold(B, N, R, cold, idx, cnt, cap, hot, st)
    side.synchronize()
    assert int(st) == 0
    hc = hot.cpu().numpy()
    for b, x in enumerate(lists):
        assert np.array_equal(hc[b, : len(x)], O.gather_rows(cold[b].numpy(), x))
        assert not hc[b, len(x):].any()
    idx[1, 3] = N + 5
    lsa.lsa_gather_cold(B, N, R, cold, idx, cnt, cap, hot, st)
    torch.cuda.synchronize()
    assert int(st) == lsa.LSA_ERR_RANGE


def test_gather_many_unbalanced_sequences():
    """70 sequences with fetch counts from 0 to the whole pool (rows of 64 bytes): the
    blocks share one flat range of rows, including empty and capped sequences."""
    g = np.random.default_rng(3)
    B, N, R = 70, 3000, 64
    cold = torch.from_numpy(g.integers(0, 256, size=(B, N, R), dtype=np.uint8)).pin_memory()
    sizes = [0 if b % 7 == 0 else (N if b % 11 == 0 else int(g.integers(1, 400))) for b in range(B)]
    lists = [np.sort(g.choice(N, size=n, replace=False)) for n in sizes]
    cap = N
    idx = torch.zeros(B, cap, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    for b, x in enumerate(lists):
        idx[b, : len(x)] = torch.from_numpy(x.astype(np.int32))
        cnt[b] = len(x)
    hot = torch.zeros(B, cap, R, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.lsa_gather_cold(B, N, R, cold, idx, cnt, cap, hot, st)
    torch.cuda.synchronize()
    assert int(st) == 0
    hc = hot.cpu().numpy()
    for b, x in enumerate(lists):
        assert np.array_equal(hc[b, : len(x)], O.gather_rows(cold[b].numpy(), x)), b
        assert not hc[b, len(x):].any()


def test_gather_rejects_pageable_memory():
    cold = torch.zeros(1, 10, 16, dtype=torch.uint8)            # not pinned
    idx = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    hot = torch.zeros(1, 4, 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_gather_cold(1, 10, 16, cold, idx, cnt, 4, hot)
    assert e.value.code == lsa.LSA_ERR_INVALID_ARG
