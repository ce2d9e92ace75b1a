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


def _select_fetch(marks, cap, want_words=True):
    """lsa_select_fetch on layer marks [L][B][N] (bool); host copies of its outputs."""
    L, B, N = marks.shape
    Nw = (N + 31) // 32
    mask = torch.from_numpy(O.pack_bits(marks).view(np.int32).copy()).cuda()
    U = torch.full((B, Nw), -5, dtype=torch.int32, device="cuda") if want_words else None
    new = torch.full((L, B, Nw), -5, dtype=torch.int32, device="cuda") if want_words else None
    capd = max(cap, 1)
    idx_new = torch.full((L, B, capd), -7, dtype=torch.int32, device="cuda")
    cnt_new = torch.full((L, B), -7, dtype=torch.int32, device="cuda")
    idx_U = torch.full((B, capd), -7, dtype=torch.int32, device="cuda")
    cnt_U = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_select_fetch_workspace_bytes(B, N))
    lsa.lsa_select_fetch(B, L, N, mask, U, new, cap, idx_new, cnt_new, idx_U, cnt_U, ws, status=st)
    torch.cuda.synchronize()
    out = dict(idx_new=idx_new.cpu().numpy(), cnt_new=cnt_new.cpu().numpy(), idx_U=idx_U.cpu().numpy(),
               cnt_U=cnt_U.cpu().numpy(), status=int(st.item()))
    if want_words:
        out["U"] = C.unpack(U, N)
        out["new"] = C.unpack(new, N)
    return out


@pytest.mark.parametrize("L,B,N,cap", [(3, 5, 3000, 3000), (1, 2, 33, 33), (3, 4, 262144, 262144),
                                       (8, 3, 70001, 70001), (2, 3, 5000, 120)])
def test_select_fetch_exact(L, B, N, cap):
    """The fused union / new sets / fetch lists against the oracle's set operations, and
    the capacity report when a list overflows."""
    g = np.random.default_rng(L * 1000 + N)
    dens = g.uniform(0.0, 0.35, size=(L, B, 1))
    marks = g.random((L, B, N)) < dens
    marks[:, 0, : min(N, 40)] = True                      # a dense head and an empty tail
    if B > 2:
        marks[:, -1, :] = False
    out = _select_fetch(marks, cap)
    over = False
    for b in range(B):
        Ue, news = O.or_union([marks[l, b] for l in range(L)])
        assert np.array_equal(out["U"][b], Ue), b
        e = O.compact(Ue)
        assert out["cnt_U"][b] == e.size, b
        assert np.array_equal(out["idx_U"][b, : min(cap, e.size)], e[:cap]), b
        over |= e.size > cap
        for l in range(L):
            assert np.array_equal(out["new"][l, b], news[l]), (l, b)
            e = O.compact(news[l])
            assert out["cnt_new"][l, b] == e.size, (l, b)
            assert np.array_equal(out["idx_new"][l, b, : min(cap, e.size)], e[:cap]), (l, b)
            over |= e.size > cap
    assert out["status"] == (lsa.LSA_ERR_CAPACITY if over else 0)


def test_select_fetch_equals_the_separate_calls_without_word_outputs():
    g = np.random.default_rng(3)
    L, B, N = 3, 6, 40000
    marks = g.random((L, B, N)) < 0.12
    out = _select_fetch(marks, N, want_words=False)
    Nw = (N + 31) // 32
    U = torch.zeros(B, Nw, dtype=torch.int32, device="cuda")
    for l in range(L):
        nw = torch.zeros(B, Nw, dtype=torch.int32, device="cuda")
        lsa.lsa_select_union(B, Nw, bits_tensor(marks[l]), U, nw)
        idx = torch.full((B, N), -7, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
        lsa.lsa_compact(B, N, nw, N, idx, cnt)
        torch.cuda.synchronize()
        assert np.array_equal(cnt.cpu().numpy(), out["cnt_new"][l])
        assert np.array_equal(idx.cpu().numpy(), out["idx_new"][l])
    idx = torch.full((B, N), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    lsa.lsa_compact(B, N, U, N, idx, cnt)
    torch.cuda.synchronize()
    assert np.array_equal(cnt.cpu().numpy(), out["cnt_U"])
    assert np.array_equal(idx.cpu().numpy(), out["idx_U"])


def test_select_fetch_more_sequences_than_one_launch():
    g = np.random.default_rng(11)
    L, B, N = 2, 70000, 100
    marks = g.random((L, B, N)) < 0.2
    out = _select_fetch(marks, N)
    for b in range(0, B, 997):
        Ue, news = O.or_union([marks[l, b] for l in range(L)])
        assert np.array_equal(out["idx_U"][b, : out["cnt_U"][b]], O.compact(Ue)), b
        for l in range(L):
            assert np.array_equal(out["idx_new"][l, b, : out["cnt_new"][l, b]], O.compact(news[l])), (l, b)
    assert (out["cnt_U"] == marks.any(axis=0).sum(axis=1)).all()


@pytest.mark.parametrize("B,N,k,L", [(5, 40000, 512, 3), (3, 262144, 2048, 3), (2, 3000, 5000, 3),
                                     (4, 3001, 100, 5), (3, 7777, 64, 1)])
def test_topk_keyed_with_selection_keys_equals_topk(B, N, k, L):
    """The union's keys written by lsa_select_fetch and lsa_topk_keyed on them give
    exactly lsa_topk's result (keys over the logits of every layer) and the oracle's;
    N not a multiple of 4 reads the logits one by one, L > 3 takes the wider kernel."""
    g = np.random.default_rng(N + k)
    marks = g.random((L, B, N)) < 0.25
    logits = np.round(g.standard_normal((L, B, N)) * 4, 1).astype(np.float32)   # ties
    Nw = (N + 31) // 32
    mask = torch.from_numpy(O.pack_bits(marks).view(np.int32).copy()).cuda()
    lg = torch.from_numpy(logits).cuda()
    idx_new = torch.empty(L, B, N, dtype=torch.int32, device="cuda")
    cnt_new = torch.empty(L, B, dtype=torch.int32, device="cuda")
    idx_U = torch.empty(B, N, dtype=torch.int32, device="cuda")
    cnt_U = torch.empty(B, dtype=torch.int32, device="cuda")
    key_U = torch.empty(B, N, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_select_fetch_workspace_bytes(B, N))
    lsa.lsa_select_fetch(B, L, N, mask, None, None, N, idx_new, cnt_new, idx_U, cnt_U, ws, logit=lg, key_U=key_U)
    got = torch.full((B, k), -9, dtype=torch.int32, device="cuda")
    got_n = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    lsa.lsa_topk_keyed(B, k, idx_U, N, cnt_U, key_U, got, got_n)
    ref = torch.full((B, k), -9, dtype=torch.int32, device="cuda")
    ref_n = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    wst = lsa.workspace(lsa.lsa_topk_workspace_bytes(B, N))
    lsa.lsa_topk(B, L, N, k, idx_U, N, cnt_U, lg, ref, ref_n, wst)
    torch.cuda.synchronize()
    assert torch.equal(got, ref) and torch.equal(got_n, ref_n)
    got, got_n = got.cpu().numpy(), got_n.cpu().numpy()
    for b in range(B):
        U = marks[:, b].any(axis=0)
        fetched = O.compact(U)
        key = O.fetched_key(logits[:, b].astype(np.float64), np.ones((L, N), dtype=bool))
        want = O.topk_in_fetched(fetched, key, k)
        assert got_n[b] == want.size
        assert np.array_equal(got[b, : want.size], want), b


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


def test_topk_all_equal_long_list_and_mixed_ties():
    """600,000 equal keys (every warp's part holds more keys at the threshold than it
    records, so the output rescans the part) and a list of 20 distinct large keys among
    ties: the kept entries are the large keys and then the lowest-index ties."""
    L, B, N, k = 1, 2, 600000, 2048
    logits = np.full((L, B, N), 1.25, dtype=np.float32)
    big = np.array([7, 1000, 99999, 123456, 599999] + list(range(300000, 300015)))
    logits[0, 1, big] = 5.0 + np.arange(big.size, dtype=np.float32)
    idx = [np.arange(N), np.arange(N)]
    topk, tc = run_topk(idx, logits, k, N)
    assert tc[0] == k and np.array_equal(topk[0, :k], np.arange(k))
    want = np.sort(np.concatenate([big, np.setdiff1d(np.arange(N), big)[: k - big.size]]))
    assert tc[1] == k and np.array_equal(topk[1, :k], want)


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
