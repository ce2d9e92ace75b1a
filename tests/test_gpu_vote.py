"""Parity of lsa_vote_labels (per-layer softmax, nucleus top-p, cross-layer vote, BCE +
focal loss) with the fp64 oracle.  Entries whose nucleus membership lies within the
summation tolerance of the top-p boundary are excluded from exact comparison."""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import build
from oracle import lsa_oracle as O
from synth import workloads as W

import lsa_cases as C

pytestmark = pytest.mark.gpu

# The device sums fp32 exponentials in fp64; the oracle uses fp64 exponentials.  The
# normalised mass before an entry agrees to ~1e-7 relative, so a membership decision is
# ambiguous only when that mass lies within BAND of top_p.
BAND = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    lsa.lib()


def run_vote(x: np.ndarray, top_p, theta, scores=None, gamma=2.0):
    L, P, N = x.shape
    Nw = (N + 31) // 32
    logits = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    golden = torch.full((P, Nw), -1, dtype=torch.int32, device="cuda")
    counts = torch.full((P, N), 255, dtype=torch.uint8, device="cuda")
    sc = None if scores is None else torch.from_numpy(np.ascontiguousarray(scores, dtype=np.float32)).cuda()
    loss = torch.zeros(2, dtype=torch.float64, device="cuda")
    ws = lsa.workspace(lsa.lsa_vote_labels_workspace_bytes(L, P, N))
    lsa.lsa_vote_labels(L, P, N, logits, top_p, theta, golden, counts, sc, gamma, loss if sc is not None else None,
                        ws)
    torch.cuda.synchronize()
    return C.unpack(golden, N), counts.cpu().numpy().astype(np.int64), loss.cpu().numpy()


def oracle_rows(x, top_p):
    """Nucleus membership and ambiguity (mass before within BAND of top_p) per row."""
    L, P, N = x.shape
    sel = np.zeros((L, P, N), dtype=bool)
    amb = np.zeros((L, P, N), dtype=bool)
    for l in range(L):
        for p in range(P):
            xr = x[l, p].astype(np.float64)
            e = np.exp(xr - xr.max())
            pi = e / e.sum()
            order = np.lexsort((np.arange(N), -pi))
            before = np.cumsum(pi[order]) - pi[order]
            sel[l, p][order] = before < top_p
            amb[l, p][order] = np.abs(before - top_p) <= BAND
            assert np.array_equal(sel[l, p], O.nucleus(xr, top_p))
    return sel, amb


def check_vote(x, top_p, theta, got_golden, got_counts):
    sel, amb = oracle_rows(x, top_p)
    count = sel.sum(axis=0)
    namb = amb.sum(axis=0)
    # counts: exact where no layer is ambiguous, within the number of ambiguous layers elsewhere
    assert np.all(np.abs(got_counts - count) <= namb)
    golden = count >= theta
    sure = (namb == 0) | (count - namb >= theta) | (count + namb < theta)
    bad = (got_golden != golden) & sure
    assert not bad.any(), f"{int(bad.sum())} golden labels differ outside the band"
    assert np.array_equal(got_golden, got_counts >= theta)       # label <=> count >= theta
    return golden, sure


@pytest.mark.parametrize("N", [1000, 4096, 33])
def test_vote_random_with_ties(N):
    g = np.random.default_rng(N)
    L, P = 5, 3
    x = np.round(g.standard_normal((L, P, N)) * 3, 1).astype(np.float32)      # many ties
    gg, gc, _ = run_vote(x, 0.6, 3)
    check_vote(x, 0.6, 3, gg, gc)


@pytest.mark.parametrize("top_p", [0.1, 0.6, 0.95, 1.0])
def test_vote_top_p_range(top_p):
    g = np.random.default_rng(7)
    x = (g.standard_normal((4, 2, 3000)) * 2).astype(np.float32)
    gg, gc, _ = run_vote(x, top_p, 2)
    check_vote(x, top_p, 2, gg, gc)


@pytest.mark.parametrize("top_p", [0.1, 0.6, 0.95])
def test_vote_full_length_rows(top_p):
    """Rows of 2^17 logits: the candidate run spans from a few entries (top_p = 0.1) to a
    few thousand (top_p = 0.95)."""
    g = np.random.default_rng(int(top_p * 100))
    x = g.standard_normal((3, 2, 2 ** 17)).astype(np.float32)
    x[:, 1] *= 3.0
    gg, gc, _ = run_vote(x, top_p, 2)
    check_vote(x, top_p, 2, gg, gc)


def test_vote_dense_ties_full_length():
    """Logits on a 0.01 grid: hundreds of entries share the crossing value, so the
    crossing is resolved by sorting the whole run."""
    g = np.random.default_rng(5)
    x = np.round(g.standard_normal((3, 2, 2 ** 17)), 2).astype(np.float32)
    gg, gc, _ = run_vote(x, 0.6, 2)
    check_vote(x, 0.6, 2, gg, gc)


def test_vote_ragged_lengths_and_outliers():
    """N not a multiple of 4 (scalar loads), a late maximum far above the first block of
    logits (re-anchoring), and -inf entries."""
    g = np.random.default_rng(9)
    x = g.standard_normal((3, 2, 50001)).astype(np.float32)
    x[0, 0, 45000] = 30.0
    x[1, 1, 40000:40010] = 12.0
    x[2, :, ::7] = -np.inf
    gg, gc, _ = run_vote(x, 0.6, 1)
    check_vote(x, 0.6, 1, gg, gc)


def test_vote_all_equal_logits_exact_nucleus():
    N = 2 ** 17
    x = np.zeros((3, 2, N), dtype=np.float32)
    gg, gc, _ = run_vote(x, 0.6, 3)
    # every pi = 2^-17; the nucleus is the first ceil(0.6 N) = 78644 entries of every row
    assert np.all(gc[:, :78644] == 3) and np.all(gc[:, 78644:] == 0)
    assert gg[:, :78644].all() and not gg[:, 78644:].any()


def test_vote_one_hot_and_theta_special_cases():
    N = 5000
    x = np.zeros((4, 2, N), dtype=np.float32)
    x[:, 0, 17] = 60.0
    x[:, 1, 4999] = 60.0
    gg, gc, _ = run_vote(x, 0.6, 4)
    assert np.flatnonzero(gg[0]).tolist() == [17] and np.flatnonzero(gg[1]).tolist() == [4999]
    g = np.random.default_rng(3)
    x = (g.standard_normal((4, 2, 1000)) * 2).astype(np.float32)
    g1, c1, _ = run_vote(x, 0.6, 1)
    sel, amb = oracle_rows(x, 0.6)
    sure = ~amb.any(axis=0)
    assert np.array_equal(g1[sure], sel.any(axis=0)[sure])           # theta = 1: OR of nuclei
    g5, _, _ = run_vote(x, 0.6, 5)
    assert not g5.any()                                              # theta > L: no label


def test_vote_full_size_every_position():
    """The full vote workload (24 layers x 64 positions x 2^17 logits) in one call; every
    position's counts and labels against the oracle (positions checked on a thread pool)."""
    v = W.VOTE_WORKLOADS["vote_labels_l24_p64_n131072"]
    x = torch.empty(v.L, v.P, v.N, dtype=torch.float32, device="cuda")
    for p in range(v.P):
        bs = W.vote_boost_set(v, p, "cuda")
        for l in range(v.L):
            x[l, p] = W.vote_logits(v, l, p, "cuda", boost_set=bs)
    Nw = (v.N + 31) // 32
    golden = torch.zeros(v.P, Nw, dtype=torch.int32, device="cuda")
    counts = torch.zeros(v.P, v.N, dtype=torch.uint8, device="cuda")
    ws = lsa.workspace(lsa.lsa_vote_labels_workspace_bytes(v.L, v.P, v.N))
    lsa.lsa_vote_labels(v.L, v.P, v.N, x, v.top_p, v.theta, golden, counts, None, v.gamma, None, ws)
    torch.cuda.synchronize()
    x_h = x.cpu().numpy()
    g_h = C.unpack(golden, v.N)
    c_h = counts.cpu().numpy().astype(np.int64)

    def one(p):
        golden_o, _ = check_vote(x_h[:, p:p + 1], v.top_p, v.theta, g_h[p:p + 1], c_h[p:p + 1])
        # the boosted entries (shared by >= 3 layers) dominate the labels
        bs = W.vote_boost_set(v, p).numpy()
        assert golden_o[0, bs].mean() > 0.9, p
        return p

    with ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
        assert sorted(ex.map(one, range(v.P))) == list(range(v.P))


def test_vote_loss_parity():
    """Loss against sigmoid scores of the 512K workload's scorer (sequence 0, layer 0),
    one hidden state per query position; scores computed by the oracle."""
    v = W.VOTE_WORKLOADS["vote_labels_l24_p64_n131072"]
    w = W.scaled(W.WORKLOADS["lsa_step_512k_b8_bf16"], B=1, L=1, N=4096)
    P, L, N = 8, 6, w.N
    bias, direction = W.load_params(w.name)
    Wd, Wu, Ww = (t[0] for t in W.all_layer_weights(W.WORKLOADS["lsa_step_512k_b8_bf16"]))
    hp = W.position_hidden(W.VOTE_WORKLOADS["vote_labels_l24_p64_n131072"], w)[:P]
    K = W.keys(w, 0, 0, direction[0, 0].double(), 0, N)[0]
    from oracle import step as OS
    scores = np.zeros((P, N))
    for p in range(P):
        q, wv = OS.project(C.raw(hp[p]), C.raw(Wd), C.raw(Wu), C.raw(Ww), w.H, w.dI, "bf16")
        z, I, _ = OS.score_layer(q, wv, float(bias[0]), C.raw(K), None, "bf16")
        scores[p] = I
    scores = scores.astype(np.float32)
    g = np.random.default_rng(11)
    x = (g.standard_normal((L, P, N)) * 2).astype(np.float32)
    boost = g.random((P, N)) < 0.05
    x[:3] += np.where(boost, 5.0, 0.0)[None]
    gg, gc, loss = run_vote(x, v.top_p, v.theta, scores, v.gamma)
    golden, sure = check_vote(x, v.top_p, v.theta, gg, gc)
    assert sure.all(), "loss test inputs must have no ambiguous labels"
    bce, fl = O.bce_focal(scores.astype(np.float64), golden, v.gamma)
    assert loss[0] == pytest.approx(bce, rel=1e-5)
    assert loss[1] == pytest.approx(fl, rel=1e-5)
    assert math.isfinite(loss[0]) and loss[0] > 0
