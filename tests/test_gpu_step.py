"""The whole indexer step at the 1M-context size (B = 32 sequences of N = 262,144 entries,
three layers, e4m3 keys, top-k 2048), run by the benchmark's own step object in the launch
configuration it times: the projection, all layers scored in one launch, the incremental
union and the compactions, the top-k inside the fetched set, and the gathers on the side
stream.

The scores themselves are held to the oracle in the score tests.  Here the step's own
logits and masks decide every float comparison, and everything downstream is integer or
byte work, so it is held bit for bit to the oracle's set operations applied to them:
masks against the logits' signs, the union and new-sets, the fetch lists and counts, the
top-k sets of all sequences, and the gathered rows byte for byte."""
import numpy as np
import pytest
import torch

import bench
import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import build
from oracle import lsa_oracle as O
from synth import workloads as W

import lsa_cases as C

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    lsa.lib()


def test_full_step_1m_b32_fp8_selection_exact():
    w = W.WORKLOADS["lsa_step_1m_b32_fp8"]
    dev = torch.device("cuda")
    inp = bench.device_inputs(w, dev)
    cold = bench.cold_pool(w, dev)
    trig = bench.Trigger(lsa, w, inp, cold, dev)
    trig.run()
    torch.cuda.synchronize()
    assert int(trig.status.item()) == 0
    L, B, N, k = w.L, w.B, w.N, w.k

    logit = trig.logit.cpu().numpy()                       # [L][B][N] fp32
    mark = C.unpack(trig.mask, N)                          # [L][B][N]
    assert np.array_equal(mark, logit >= 0)                # I >= 0.5  <=>  z >= 0
    frac = mark.mean()
    assert 0.02 < frac < 0.3, frac

    U, news = O.or_union([mark[l] for l in range(L)])      # elementwise over [B][N]
    assert np.array_equal(C.unpack(trig.U, N), U)
    new_bits = C.unpack(trig.new, N)
    for l in range(L):
        assert np.array_equal(new_bits[l], news[l]), l

    cnt_new = trig.cnt_new.cpu().numpy()
    idx_new = trig.idx_new.cpu().numpy()
    cnt_U = trig.cnt_U.cpu().numpy()
    idx_U = trig.idx_U.cpu().numpy()
    topk = trig.topk.cpu().numpy()
    topk_cnt = trig.topk_cnt.cpu().numpy()
    for b in range(B):
        for l in range(L):
            e = O.compact(news[l][b])
            assert cnt_new[l, b] == len(e), (l, b)
            assert np.array_equal(idx_new[l, b, : len(e)], e), (l, b)
        fetched = O.compact(U[b])
        assert cnt_U[b] == len(fetched), b
        assert np.array_equal(idx_U[b, : len(fetched)], fetched), b
        key = O.fetched_key(logit[:, b].astype(np.float64), mark[:, b])
        expect = O.topk_in_fetched(fetched, key, k)
        assert topk_cnt[b] == len(expect) == min(k, len(fetched)), b
        assert np.array_equal(topk[b, : len(expect)], expect), b
        assert (topk[b, len(expect):] == -1).all(), b

    # gathered rows: every row of three sequences in every layer
    cold_np = cold.numpy()
    for b in (0, 13, B - 1):
        for l in range(L):
            n = int(cnt_new[l, b])
            got = trig.hot[l, b, :n].cpu().numpy()
            assert np.array_equal(got, O.gather_rows(cold_np[b], idx_new[l, b, :n])), (l, b)
