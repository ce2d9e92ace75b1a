"""lsa_topk_noalloc -- the top-k variant for callers that cannot allocate device memory
at call time (its scratch is a built-in device array) -- gives the same result as
lsa_topk with a caller workspace, on two calls in a row, through the C ABI."""
import numpy as np
import pytest
import torch

import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    lsa.lib()


def _case(seed, B, L, N, cap):
    g = np.random.default_rng(seed)
    logit = torch.from_numpy(np.round(g.standard_normal((L, B, N)) * 4, 1).astype(np.float32)).cuda()
    idx = torch.full((B, cap), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    for b in range(B):
        n = int(g.integers(0, cap + 1))
        idx[b, :n] = torch.from_numpy(np.sort(g.choice(N, size=n, replace=False)).astype(np.int32))
        cnt[b] = n
    return logit, idx, cnt


def _both(B, L, N, k, cap, logit, idx, cnt):
    ref = torch.full((B, k), -9, dtype=torch.int32, device="cuda")
    ref_n = torch.full((B,), -9, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_topk_workspace_bytes(B, cap))
    lsa.lsa_topk(B, L, N, k, idx, cap, cnt, logit, ref, ref_n, ws)
    got = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    got_n = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    lsa.lsa_topk_noalloc(B, L, N, k, idx, cap, cnt, logit, got, got_n)
    torch.cuda.synchronize()
    return ref, ref_n, got, got_n


def test_noalloc_matches_workspace_variant_twice():
    B, L, N, cap, k = 8, 3, 40000, 20000, 512
    for seed in (1, 2):      # the second call runs over the first call's leftover scratch
        logit, idx, cnt = _case(seed, B, L, N, cap)
        ref, ref_n, got, got_n = _both(B, L, N, k, cap, logit, idx, cnt)
        assert torch.equal(got_n, ref_n)
        assert torch.equal(got, ref)
        assert int(ref_n.max()) == k      # the case exercises the radix select, not only n <= k


def test_noalloc_rejects_sizes_beyond_its_scratch():
    B, cap = 33, 262144          # 8,650,752 slots > 2^23
    idx = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(lsa.LsaError) as e:
        lsa.lsa_topk_noalloc(B, 1, 16, 4, idx, cap, idx, idx, idx, None)
    assert e.value.code == lsa.LSA_ERR_NOMEM
