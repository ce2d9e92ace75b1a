"""lsa_topk_noalloc -- the top-k variant for callers that cannot allocate device memory
at call time (its scratch is a built-in device array) -- gives the same result as
lsa_topk with a caller workspace, on two calls in a row, through the C ABI.

The large case puts every sequence's candidate slice beyond what one CTA keeps in shared
memory, so the kernel really reads and writes the built-in array, and it fills that array
exactly (B * cap = 2^23 slots).  Both cases also compare with the oracle's top-k."""

import numpy as np
import pytest
import torch

import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import build
from oracle import lsa_oracle as O

pytestmark = pytest.mark.gpu

SCRATCH_SLOTS = 1 << 23          # the array's size in uint32 slots, as include/lsa.h states


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    lsa.lib()


def _case(seed, B, L, N, cap, lo=0):
    """Logits rounded to 0.1 (many equal keys) and per-sequence fetch lists of
    lo..cap ascending entries."""
    g = np.random.default_rng(seed)
    logit_np = np.round(g.standard_normal((L, B, N)) * 4, 1).astype(np.float32)
    idx_np = np.full((B, cap), -1, dtype=np.int32)
    cnt_np = np.zeros(B, dtype=np.int32)
    for b in range(B):
        n = int(g.integers(lo, cap + 1))
        idx_np[b, :n] = np.sort(g.choice(N, size=n, replace=False)).astype(np.int32)
        cnt_np[b] = n
    return (logit_np, idx_np, cnt_np, torch.from_numpy(logit_np).cuda(), torch.from_numpy(idx_np).cuda(),
            torch.from_numpy(cnt_np).cuda())


def _both(B, L, N, k, cap, logit, idx, cnt):
    ref = torch.full((B, k), -9, dtype=torch.int32, device="cuda")
    ref_n = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_topk_workspace_bytes(B, cap))
    lsa.lsa_topk(B, L, N, k, idx, cap, cnt, logit, ref, ref_n, ws)
    got = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    got_n = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    lsa.lsa_topk_noalloc(B, L, N, k, idx, cap, cnt, logit, got, got_n)
    torch.cuda.synchronize()
    return ref.cpu().numpy(), ref_n.cpu().numpy(), got.cpu().numpy(), got_n.cpu().numpy()


def _check_against_oracle(logit_np, idx_np, cnt_np, k, got, got_n, seqs):
    """The oracle's top-k of the fetched entries keyed by their largest logit over the
    layers (the same fp32 values, compared exactly in fp64)."""
    for b in seqs:
        n = int(cnt_np[b])
        key = logit_np[:, b, :].astype(np.float64).max(axis=0)
        want = O.topk_in_fetched(idx_np[b, :n], key, k)
        assert int(got_n[b]) == want.size, b
        assert np.array_equal(got[b, : want.size], want), b
        assert (got[b, want.size:] == -1).all(), b


def test_noalloc_matches_workspace_variant_twice():
    B, L, N, cap, k = 8, 3, 40000, 20000, 512
    for seed in (1, 2):      # the second call runs over the first call's leftover scratch
        logit_np, idx_np, cnt_np, logit, idx, cnt = _case(seed, B, L, N, cap)
        ref, ref_n, got, got_n = _both(B, L, N, k, cap, logit, idx, cnt)
        assert np.array_equal(got_n, ref_n)
        assert np.array_equal(got, ref)
        assert int(ref_n.max()) == k      # the case exercises the radix select, not only n <= k
        _check_against_oracle(logit_np, idx_np, cnt_np, k, got, got_n, range(B))


def test_noalloc_uses_the_whole_scratch_array_twice():
    """B = 16, cap = 2^19: B * cap is the array's full size, and each sequence's slice per
    CTA (up to 8 CTAs per sequence: 65,536 candidates) exceeds the shared-memory slice of
    32,768 keys, so the keys live in the built-in array.  Two calls with different inputs
    in a row: the second runs over the first one's leftovers."""
    B, L, N, cap, k = 16, 3, 600000, 1 << 19, 2048
    assert B * cap == SCRATCH_SLOTS
    for seed in (3, 4):
        logit_np, idx_np, cnt_np, logit, idx, cnt = _case(seed, B, L, N, cap, lo=cap - 30000)
        assert int(cnt_np.min()) > 8 * 32768          # the key slices go to the array
        ref, ref_n, got, got_n = _both(B, L, N, k, cap, logit, idx, cnt)
        assert np.array_equal(got_n, ref_n)
        assert np.array_equal(got, ref)
        assert (ref_n == k).all()
        _check_against_oracle(logit_np, idx_np, cnt_np, k, got, got_n, (0, 7, 15))


def test_noalloc_rejects_sizes_beyond_its_scratch_and_clears_the_last_error():
    B, cap = 33, 262144          # 8,650,752 slots > 2^23
    idx = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_topk_noalloc(B, 1, 16, 4, idx, cap, idx, idx, idx, None)
    assert e.value.code == lsa.LSA_ERR_NOMEM
    assert lsa.lib().lsa_last_error().decode() != ""
    # a successful call afterwards leaves no stale message behind
    logit_np, idx_np, cnt_np, logit, idx2, cnt = _case(5, 2, 1, 1000, 100)
    out = torch.empty((2, 8), dtype=torch.int32, device="cuda")
    out_n = torch.empty(2, dtype=torch.int32, device="cuda")
    lsa.lsa_topk_noalloc(2, 1, 1000, 8, idx2, 100, cnt, logit, out, out_n)
    torch.cuda.synchronize()
    assert lsa.lib().lsa_last_error().decode() == ""
