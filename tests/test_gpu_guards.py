"""Out-of-bounds writes would go unseen without a sanitizer, so outputs here live between
two 4 KB canary regions that must be intact after each call (ragged sizes throughout)."""
import numpy as np
import pytest
import torch

import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import build
from oracle import lsa_oracle as O

import lsa_cases as C

pytestmark = pytest.mark.gpu
GUARD = 4096
CANARY = 0x5A


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    lsa.lib()


class Guarded:
    """A device tensor of `shape` and `dtype` with canary bytes on both sides."""

    def __init__(self, shape, dtype, fill=0):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.raw = torch.full((GUARD + n + GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD: GUARD + n].view(dtype).reshape(shape)
        self.t.fill_(fill)

    def intact(self):
        r = self.raw.cpu().numpy()
        return bool((r[:GUARD] == CANARY).all() and (r[-GUARD:] == CANARY).all())


def test_guards_compact_topk_union():
    g = np.random.default_rng(1)
    B, N, cap, L, k = 3, 1001, 700, 2, 37
    marks = g.random((L, B, N)) < np.array([0.2, 0.5])[:, None, None]
    masks = torch.from_numpy(O.pack_bits(marks.reshape(L * B, N)).view(np.int32).reshape(L, B, -1)).cuda()
    Nw = masks.shape[-1]
    U = Guarded((B, Nw), torch.int32)
    new = Guarded((B, Nw), torch.int32)
    for l in range(L):
        lsa.lsa_select_union(B, Nw, masks[l], U.t, new.t)
    idx = Guarded((B, cap), torch.int32, -7)
    cnt = Guarded((B,), torch.int32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.lsa_compact(B, N, U.t, cap, idx.t, cnt.t, st)
    logit = torch.from_numpy(g.standard_normal((L, B, N)).astype(np.float32)).cuda()
    topk = Guarded((B, k), torch.int32)
    tcnt = Guarded((B,), torch.int32)
    ws = Guarded((lsa.lsa_topk_workspace_bytes(B, cap),), torch.uint8)
    lsa.lsa_topk(B, L, N, k, idx.t, cap, cnt.t, logit, topk.t, tcnt.t, ws.t)
    torch.cuda.synchronize()
    for x in (U, new, idx, cnt, topk, tcnt, ws):
        assert x.intact()
    union = marks.any(axis=0)
    over = [len(O.compact(union[b])) > cap for b in range(B)]
    assert int(st.item()) == (lsa.LSA_ERR_CAPACITY if any(over) else 0)


def test_guards_gather_and_hot_pool():
    g = np.random.default_rng(2)
    B, N, R, cap, slots = 3, 999, 48, 333, 301
    cold = torch.from_numpy(g.integers(0, 256, size=(B, N, R), dtype=np.uint8)).pin_memory()
    lists = [np.sort(g.choice(N, size=n, replace=False)) for n in (0, 150, 333)]
    idx = torch.zeros(B, cap, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    for b, x in enumerate(lists):
        idx[b, : len(x)] = torch.from_numpy(x.astype(np.int32))
        cnt[b] = len(x)
    hot = Guarded((B, cap, R), torch.uint8)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.lsa_gather_cold(B, N, R, cold, idx, cnt, cap, hot.t, st)
    torch.cuda.synchronize()
    assert hot.intact() and int(st.item()) == 0
    # residency: two triggers into a pool of `slots` rows
    state = Guarded((lsa.lsa_hot_pool_state_bytes(B, N, slots),), torch.uint8)
    ws = Guarded((lsa.lsa_hot_pool_workspace_bytes(B, N, slots),), torch.uint8)
    hp = Guarded((B, slots, R), torch.uint8)
    moved = Guarded((B,), torch.int32)
    lsa.lsa_hot_pool_reset(B, N, slots, state.t)
    for t in (1, 2):
        marks = g.random((B, N)) < 0.25
        U = torch.from_numpy(O.pack_bits(marks).view(np.int32)).cuda()
        lsa.lsa_hot_pool_update(B, N, slots, R, t, U, cold, hp.t, state.t, moved.t, st, ws.t)
    torch.cuda.synchronize()
    for x in (state, ws, hp, moved):
        assert x.intact()


def test_guards_vote():
    g = np.random.default_rng(3)
    L, P, N = 4, 3, 1001
    x = torch.from_numpy((g.standard_normal((L, P, N)) * 2).astype(np.float32)).cuda()
    Nw = (N + 31) // 32
    golden = Guarded((P, Nw), torch.int32)
    counts = Guarded((P, N), torch.uint8)
    scores = torch.from_numpy(g.random((P, N)).astype(np.float32)).cuda()
    loss = Guarded((2,), torch.float64)
    ws = Guarded((lsa.lsa_vote_labels_workspace_bytes(L, P, N),), torch.uint8)
    lsa.lsa_vote_labels(L, P, N, x, 0.6, 2, golden.t, counts.t, scores, 2.0, loss.t, ws.t)
    torch.cuda.synchronize()
    for t in (golden, counts, loss, ws):
        assert t.intact()
    assert not (C.unpack(golden.t, N) != (counts.t.cpu().numpy() >= 2)).any()


@pytest.mark.parametrize("wname,N", [("lsa_step_16k_tiny_fp32", 1001), ("lsa_step_128k_b1_bf16", 5000)])
def test_guards_score(wname, N):
    w = C.W.scaled(C.W.WORKLOADS[wname], N=N)
    inp = C.make_inputs(w)
    B, L = w.B, w.L
    Nw = (N + 31) // 32
    mask = Guarded((L, B, Nw), torch.int32)
    logit = Guarded((L, B, N), torch.float32)
    score = Guarded((L, B, N), torch.float32)
    q = Guarded((L, B, w.H, w.dI), inp.h.dtype)
    wv = Guarded((L, B, w.H), torch.float32)
    ws = Guarded((lsa.lsa_index_score_workspace_bytes(B, L, N, w.D, w.r, w.H, w.dI, lsa.dtype_code(inp.h),
                                                      lsa.dtype_code(inp.K)),), torch.uint8)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.lsa_index_score(B, L, N, w.D, w.r, w.H, w.dI, lsa.dtype_code(inp.h), inp.h, inp.Wd, inp.Wu, inp.Ww,
                        inp.bias, lsa.dtype_code(inp.K), inp.K, inp.kscale, -1, None, None, q.t, wv.t,
                        mask.t, logit.t, score.t, ws.t, status=st)
    torch.cuda.synchronize()
    for t in (mask, logit, score, q, wv, ws):
        assert t.intact()
    assert int(st.item()) == 0
