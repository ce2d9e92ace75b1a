"""Pins of the fp64 oracle against facts fixed outside the oracle itself: a hand-derived
worked example, closed forms, library routines for the number formats, invariants the
pages state, and independent brute-force formulations on tiny inputs."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lsa_oracle as O
from oracle import step as OS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- formats

def test_decode_bf16_matches_torch_for_every_pattern():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = O.decode_bf16(pats)
    ref = torch.from_numpy(pats.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_decode_e4m3_spec_values_and_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.decode_e4m3(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    assert ((ours == ref) | (np.isnan(ours) & np.isnan(ref))).all()
    # OCP E4M3: max normal 448 = 1.75 * 2**8, min subnormal 2**-9, S.1111.111 = NaN
    assert ours[0x7E] == 448.0 and ours[0xFE] == -448.0
    assert ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    assert ours[0x38] == 1.0


def test_round_to_bf16_ties_to_even_and_torch():
    one = 1.0
    assert O.round_to_bf16(one + 2 ** -8) == 1.0                 # tie -> even mantissa 0
    assert O.round_to_bf16(one + 3 * 2 ** -8) == one + 2 ** -6   # tie -> even mantissa 2
    assert O.round_to_bf16(one + 2 ** -8 + 2 ** -30) == one + 2 ** -7
    assert O.round_to_bf16(2.0 ** -133) == 2.0 ** -133            # smallest subnormal
    assert O.round_to_bf16(2.0 ** -134) == 0.0                    # tie below it -> 0 (even)
    g = np.random.default_rng(7)
    x = (g.standard_normal(200000) * np.exp2(g.integers(-130, 120, 200000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert (O.round_to_bf16(x.astype(np.float64)) == ref).all()


# ----------------------------------------------------------------------------- worked example

def _worked():
    with open(os.path.join(GOLDEN, "score_worked_example.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("bf16", [False, True])
def test_worked_example_projection_and_score(bf16):
    ex = _worked()
    e = ex["expected"]
    q, w = O.project_query(ex["h"], ex["W_down"], ex["W_up"], ex["W_w"], ex["H"], ex["dI"], bf16)
    assert np.array_equal(q, np.array(e["q"])) and np.array_equal(w, np.array(e["w"]))
    z = O.head_fused_logits(q, w, ex["bias"], ex["K"])
    assert np.array_equal(z, np.array(e["z"]))
    assert np.array_equal(O.threshold_mark(z), np.array(e["mark"]))
    np.testing.assert_allclose(O.sigmoid(z), 1 / (1 + np.exp(-np.array(e["z"]))), rtol=0, atol=0)


def test_projection_rounds_c_before_the_up_projection():
    """bf16 boundaries: c = h W_down is rounded to bf16 before q = c W_up.  With
    c = [1 + 3 * 2^-9, 1] (0.75 of a bf16 ulp above 1: rounds up to 1 + 2^-7) and
    W_up = [1, -1]^T, q = RNE(1 + 2^-7 - 1) = 2^-7; without the rounding of c it would be
    3 * 2^-9.  In fp32 mode nothing is rounded."""
    h = np.array([1.0, 0.0])
    W_down = np.array([[1.0 + 3 * 2.0 ** -9, 1.0], [0.0, 0.0]])
    W_up = np.array([[1.0], [-1.0]])
    W_w = np.array([[2.0], [0.0]])
    q, w = O.project_query(h, W_down, W_up, W_w, 1, 1, True)
    assert q.tolist() == [[2.0 ** -7]] and w.tolist() == [2.0]
    q, w = O.project_query(h, W_down, W_up, W_w, 1, 1, False)
    assert q.tolist() == [[3 * 2.0 ** -9]]
    # the same through raw storage: a bf16 model gets the bf16 boundaries, an fp32 model
    # none (h = [1, 1] and W_down = [[1, 1], [3 * 2^-9, 0]] are bf16 values with the same c)
    h2 = np.array([1.0, 1.0])
    Wd2 = np.array([[1.0, 1.0], [3 * 2.0 ** -9, 0.0]])
    def bits(a):
        return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q, w = OS.project(bits(h2), bits(Wd2), bits(W_up), bits(W_w), 1, 1, "bf16")
    assert q.tolist() == [[2.0 ** -7]] and w.tolist() == [2.0]
    f32 = lambda a: np.asarray(a, dtype=np.float32)
    q, w = OS.project(f32(h2), f32(Wd2), f32(W_up), f32(W_w), 1, 1, "f32")
    assert q.tolist() == [[3 * 2.0 ** -9]]


def test_worked_example_through_raw_buffers():
    """The same example through the raw-storage path (bf16 bit patterns)."""
    ex = _worked()
    def bits(a):
        return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q, w = OS.project(bits(ex["h"]), bits(ex["W_down"]), bits(ex["W_up"]), bits(ex["W_w"]), 2, 2, "bf16")
    z, I, mark = OS.score_layer(q, w, ex["bias"], bits(ex["K"]), None, "bf16")
    assert np.array_equal(z, np.array(ex["expected"]["z"]))


# ----------------------------------------------------------------------------- score closed forms

def test_single_head_unit_weight_reduces_to_dot_threshold():
    """H=1, w=1: z = ReLU(q.k) + b, so with b = -t < 0 an entry is marked iff q.k >= t
    (with b = 0 every entry would be marked, since ReLU >= 0)."""
    g = np.random.default_rng(1)
    q = g.standard_normal((1, 16))
    K = g.standard_normal((500, 16))
    z0 = O.head_fused_logits(q, [1.0], 0.0, K)
    assert O.threshold_mark(z0).all()
    t = 0.75
    z = O.head_fused_logits(q, [1.0], -t, K)
    dots = np.array([sum(q[0][i] * K[s][i] for i in range(16)) for s in range(500)])
    np.testing.assert_array_equal(O.threshold_mark(z), dots >= t)
    np.testing.assert_allclose(z, np.where(dots > 0, dots, 0.0) - t, rtol=1e-13, atol=1e-13)


def test_parallel_and_antiparallel_keys_closed_form():
    g = np.random.default_rng(2)
    H, d = 4, 8
    q = g.standard_normal((H, d))
    w = g.standard_normal(H)
    # k = alpha * q_0 with q_1.. orthogonalised away -> z = w_0 * alpha * |q_0|^2 + b
    qo = q.copy()
    for h in range(1, H):
        qo[h] -= (qo[h] @ qo[0]) / (qo[0] @ qo[0]) * qo[0]
    for alpha in (0.5, 3.0):
        z = O.head_fused_logits(qo, w, 0.25, alpha * qo[0][None, :])
        assert z[0] == pytest.approx(w[0] * alpha * (qo[0] @ qo[0]) + 0.25, rel=1e-12)
        z = O.head_fused_logits(qo, w, 0.25, -alpha * qo[0][None, :])
        assert z[0] == pytest.approx(0.25, abs=1e-12)


def test_orthogonal_key_gives_bias_and_positive_homogeneity():
    g = np.random.default_rng(3)
    q = np.zeros((3, 6))
    q[:, :3] = g.standard_normal((3, 3))
    K = np.zeros((10, 6))
    K[:, 3:] = g.standard_normal((10, 3))
    z = O.head_fused_logits(q, [1.0, -2.0, 0.5], -1.5, K)
    assert np.all(z == -1.5)
    q = g.standard_normal((5, 6))
    w = g.standard_normal(5)
    K = g.standard_normal((40, 6))
    z1 = O.head_fused_logits(q, w, 0.0, K)
    z3 = O.head_fused_logits(q, w, 0.0, 3.0 * K)
    np.testing.assert_allclose(z3, 3.0 * z1, rtol=1e-12, atol=1e-12)


def test_score_brute_force_loops():
    """Independent formulation: explicit loops over (entry, head, component)."""
    g = np.random.default_rng(4)
    H, d, n = 3, 5, 12
    q = g.standard_normal((H, d))
    w = g.standard_normal(H)
    K = g.standard_normal((n, d))
    b = 0.3
    for s in range(n):
        acc = b
        for h in range(H):
            dot = 0.0
            for i in range(d):
                dot += q[h][i] * K[s][i]
            if dot > 0:
                acc += w[h] * dot
        assert O.head_fused_logits(q, w, b, K)[s] == pytest.approx(acc, rel=1e-12, abs=1e-12)


def test_threshold_boundary_and_sigmoid():
    assert O.sigmoid(0.0) == 0.5
    assert O.threshold_mark(np.array([0.0, -1e-300, 1e-300])).tolist() == [True, False, True]
    assert O.sigmoid(np.log(3.0)) == pytest.approx(0.75, rel=1e-15)


def test_e4m3_scale_applied_per_entry():
    codes = np.array([[0x38, 0x40], [0xB8, 0x00]], dtype=np.uint8)    # [1, 2], [-1, 0]
    K = OS.decode_keys(codes, np.array([0.5, 4.0], dtype=np.float32), "e4m3")
    np.testing.assert_array_equal(K, [[0.5, 1.0], [-4.0, 0.0]])


# ----------------------------------------------------------------------------- bit sets

def test_pack_bits_order_and_padding():
    mark = np.zeros(70, dtype=bool)
    mark[[0, 31, 33, 69]] = True
    words = O.pack_bits(mark)
    assert words.tolist() == [0x80000001, 0x2, 0x20]
    assert np.array_equal(O.unpack_bits(words, 70), mark)


def test_union_and_new_sets_brute_force_and_invariants():
    g = np.random.default_rng(5)
    for _ in range(50):
        n = int(g.integers(1, 40))
        marks = [g.random(n) < g.random() for _ in range(3)]
        U, news = O.or_union(marks)
        sets = [set(np.flatnonzero(m)) for m in marks]
        assert set(np.flatnonzero(U)) == sets[0] | sets[1] | sets[2]
        seen = set()
        for m, nw in zip(sets, news):
            assert set(np.flatnonzero(nw)) == m - seen
            seen |= m
        for m in marks:                                  # union contains each layer's mask
            assert np.all(U[m])
        assert sum(int(x.sum()) for x in news) == int(U.sum())   # new sets partition U


def test_compact_brute_force():
    g = np.random.default_rng(6)
    for n in (0, 1, 31, 32, 33, 100):
        m = g.random(n) < 0.3
        idx = O.compact(m)
        assert idx.tolist() == [i for i in range(n) if m[i]]
        assert len(idx) == int(m.sum())                  # fetched count == popcount


# ----------------------------------------------------------------------------- top-k

def _topk_brute(idx, key, k):
    """s is kept iff fewer than k candidates beat it (larger key, or equal key and lower index)."""
    out = []
    for s in idx:
        beaten = sum(1 for t in idx if key[t] > key[s] or (key[t] == key[s] and t < s))
        if beaten < k:
            out.append(s)
    return sorted(out)


def test_topk_brute_force_with_ties():
    g = np.random.default_rng(8)
    for _ in range(200):
        n = int(g.integers(1, 30))
        key = np.round(g.standard_normal(40), 1)          # many ties
        idx = np.sort(g.choice(40, size=n, replace=False))
        k = int(g.integers(0, 35))
        got = O.topk_in_fetched(idx, key, k)
        assert got.tolist() == _topk_brute(idx.tolist(), key, k)
        assert set(got.tolist()) <= set(idx.tolist())    # top-k inside the fetched set
        assert len(got) == min(k, n)


def test_fine_topk_brute_force_loops():
    """The native-indexer fine selection written out with loops on tiny inputs: per
    fetched entry sum_h w_h max(0, sum_d q_hd k_d); the top-k of those among the fetched
    entries only (ties to the lower index), in ascending entry order."""
    g = np.random.default_rng(21)
    for _ in range(60):
        N, H, dI = int(g.integers(1, 25)), int(g.integers(1, 4)), int(g.integers(1, 5))
        q = np.round(g.standard_normal((H, dI)), 1)
        w = np.round(g.standard_normal(H), 1)
        K = np.round(g.standard_normal((N, dI)), 1)
        n = int(g.integers(0, N + 1))
        fetched = np.sort(g.choice(N, size=n, replace=False))
        k = int(g.integers(0, N + 2))
        scores = [sum(w[h] * max(0.0, sum(q[h, d] * K[e, d] for d in range(dI))) for h in range(H)) for e in fetched]
        got = O.fine_index_scores(q, w, K, fetched)
        assert np.allclose(got, scores, rtol=1e-12, atol=1e-12)
        key = {int(e): sc for e, sc in zip(fetched, got)}
        want = sorted(e for e in key if sum(1 for t in key if key[t] > key[e] or (key[t] == key[e] and t < e)) < k)
        assert O.fine_topk(q, w, K, fetched, k).tolist() == want


def test_fine_topk_ignores_entries_outside_the_fetched_set():
    """An entry that was not fetched is never chosen, whatever its score would be; the
    fine query, not any other, decides the order."""
    K = np.array([[10.0, 0.0], [1.0, 0.0], [0.0, 1.0], [0.0, 3.0]])
    q = np.array([[1.0, 0.0]])
    w = np.array([1.0])
    assert O.fine_topk(q, w, K, [1, 2, 3], 1).tolist() == [1]       # entry 0 (score 10) not fetched
    q2 = np.array([[0.0, 1.0]])
    assert O.fine_topk(q2, w, K, [1, 2, 3], 1).tolist() == [3]
    assert O.fine_topk(q2, w, K, [1, 2, 3], 2).tolist() == [2, 3]
    # |fetched| <= k: everything fetched, in ascending order
    assert O.fine_topk(q, w, K, [3, 1], 5).tolist() == [1, 3]
    # a negative head weight ranks larger dot products lower; ReLU zeroes negative dots
    assert O.fine_index_scores(np.array([[1.0, 1.0]]), np.array([-2.0]), K, [0, 3]).tolist() == [-20.0, -6.0]
    assert O.fine_index_scores(np.array([[-1.0, 0.0]]), np.array([1.0]), K, [0, 1]).tolist() == [0.0, 0.0]


def test_fetched_key_is_max_over_marking_layers():
    z = np.array([[1.0, -2.0, 0.5], [3.0, -1.0, -0.2], [-5.0, 0.0, 0.7]])
    m = z >= 0
    assert O.fetched_key(z, m).tolist() == [3.0, 0.0, 0.7]
    # the key follows the marks, not the largest logit: a layer that did not mark the
    # entry does not count even where its logit is larger; an unmarked entry has no key
    z = np.array([[5.0, 1.0, 2.0], [7.0, 2.0, 3.0]])
    m = np.array([[True, True, False], [False, True, False]])
    assert O.fetched_key(z, m).tolist() == [5.0, 2.0, -np.inf]


def test_fetched_key_equals_the_largest_logit_when_marks_are_the_threshold():
    """With the marks the threshold makes (z >= 0), a layer that does not mark an entry has
    a logit below every marking layer's, so for every fetched entry the key over the
    marking layers equals the largest logit over all layers (the form the fused selection
    computes its keys in); entries no layer marks have no key."""
    g = np.random.default_rng(11)
    z = np.round(g.standard_normal((4, 5000)) * 2, 1)     # ties and exact zeros included
    z[:, :10] = 0.0
    m = z >= 0
    key = O.fetched_key(z, m)
    fetched = m.any(axis=0)
    assert np.array_equal(key[fetched], z.max(axis=0)[fetched])
    assert np.all(np.isneginf(key[~fetched]))


def test_step_select_composes_the_set_operations():
    """The step's selection from per-layer marks and logits, by brute force: the top-k
    runs over the union of all layers (not one layer's new set), keyed by the largest
    logit among the marking layers."""
    g = np.random.default_rng(21)
    for _ in range(30):
        n, k = int(g.integers(1, 50)), int(g.integers(1, 12))
        z = g.standard_normal((3, n)).round(1)           # coarse values: ties happen
        marks = z >= 0.3
        out = OS.select(list(marks), z, k)
        union = [s for s in range(n) if marks[:, s].any()]
        assert out["idx_union"].tolist() == union
        seen = set()
        for l in range(3):
            new = [s for s in range(n) if marks[l, s] and s not in seen]
            assert out["idx_new"][l].tolist() == new
            seen |= set(new)
        key = {s: max(z[l, s] for l in range(3) if marks[l, s]) for s in union}
        top = sorted(s for s in union
                     if sum(1 for t in union if key[t] > key[s] or (key[t] == key[s] and t < s)) < k)
        assert out["topk"].tolist() == top


# ----------------------------------------------------------------------------- nucleus / vote

def _nucleus_brute(x, p):
    pi = np.exp(x - x.max())
    pi = pi / pi.sum()
    n = len(x)
    sel = []
    for s in range(n):
        ahead = sum(pi[t] for t in range(n) if pi[t] > pi[s] or (pi[t] == pi[s] and t < s))
        sel.append(ahead < p)
    return np.array(sel)


def test_nucleus_all_equal_logits_exact_count():
    n = 2 ** 17
    sel = O.nucleus(np.zeros(n, dtype=np.float32), 0.6)
    # every pi = 2**-17 exactly; mass before entry i is i * 2**-17 < 0.6 <=> i <= 78643
    assert int(sel.sum()) == math.ceil(0.6 * n) == 78644
    assert sel[:78644].all() and not sel[78644:].any()


def test_nucleus_stops_where_the_mass_reaches_top_p_exactly():
    # four equal logits: pi = 1/4 each (exact), masses before: 0, 1/4, 1/2, 3/4.  The
    # smallest prefix with mass >= 1/2 is the first two entries; the third has mass 1/2
    # before it, not below 1/2.
    assert O.nucleus(np.zeros(4), 0.5).tolist() == [True, True, False, False]
    assert O.nucleus(np.zeros(8), 0.25).tolist() == [True, True] + [False] * 6
    assert O.nucleus(np.zeros(8), 0.2500001).tolist() == [True, True, True] + [False] * 5


def test_nucleus_one_hot_and_two_entry_closed_form():
    x = np.zeros(1000)
    x[123] = 50.0
    assert np.flatnonzero(O.nucleus(x, 0.6)).tolist() == [123]
    for a in (-2.0, 0.0, 0.3, 0.5, 1.0, 3.0):
        p0 = 1 / (1 + math.exp(-a))                       # pi of entry 0 for logits [a, 0]
        expect = {0} if p0 >= 0.6 else ({0, 1} if p0 >= 0.4 else ({1} if (1 - p0) >= 0.6 else {0, 1}))
        if a == 0.0:
            expect = {0, 1}                               # tie -> entry 0 first (0.5 < 0.6) then 1
        assert set(np.flatnonzero(O.nucleus(np.array([a, 0.0]), 0.6)).tolist()) == expect


def test_nucleus_brute_force_with_ties():
    g = np.random.default_rng(9)
    for _ in range(100):
        n = int(g.integers(1, 25))
        x = np.round(g.standard_normal(n) * 2, 0)
        p = float(g.choice([0.1, 0.6, 0.9, 1.0]))
        assert np.array_equal(O.nucleus(x, p), _nucleus_brute(x, p))


def test_vote_special_cases():
    g = np.random.default_rng(10)
    x = g.standard_normal((5, 3, 60))
    nuclei = np.array([[O.nucleus(x[l, p], 0.6) for p in range(3)] for l in range(5)])
    golden1, count = O.vote_labels(x, 0.6, 1)
    assert np.array_equal(golden1, nuclei.any(axis=0))            # theta = 1: OR of nuclei
    golden_all, _ = O.vote_labels(x, 0.6, 5)
    assert np.array_equal(golden_all, nuclei.all(axis=0))         # theta = L: AND
    golden_none, _ = O.vote_labels(x, 0.6, 6)
    assert not golden_none.any()                                  # theta > L: nothing
    golden3, count = O.vote_labels(x, 0.6, 3)
    assert np.all(count[golden3] >= 3) and np.all(count[~golden3] < 3)
    assert np.array_equal(count, nuclei.sum(axis=0))


# ----------------------------------------------------------------------------- loss

def test_bce_focal_closed_forms():
    bce, fl = O.bce_focal([0.5, 0.5], [1, 0], 2.0)
    assert bce == pytest.approx(math.log(2), rel=1e-15)
    assert fl == pytest.approx(math.log(2) / 4, rel=1e-15)
    bce, fl = O.bce_focal([0.8, 0.2], [1, 0], 2.0)
    assert bce == pytest.approx(-math.log(0.8), rel=1e-14)
    assert fl == pytest.approx(0.04 * -math.log(0.8), rel=1e-14)
    bce, fl = O.bce_focal([1 - 1e-12, 1e-12], [1, 0], 2.0, eps=1e-15)
    assert bce == pytest.approx(1e-12, rel=1e-3)
    # clamping: a saturated wrong score costs -ln(2^-20) = 20 ln 2, not infinity
    bce, fl = O.bce_focal([0.0, 1.0], [1, 0], 2.0)
    assert bce == pytest.approx(20 * math.log(2), rel=1e-12)
    assert fl == pytest.approx((1 - 2.0 ** -20) ** 2 * 20 * math.log(2), rel=1e-12)
    bce, fl = O.bce_focal([0.9, 0.3], [1, 1], 0.0)                 # gamma = 0: FL == BCE
    assert fl == pytest.approx(bce, rel=1e-15)


# ----------------------------------------------------------------------------- gather / bias

def test_gather_rows_is_indexing():
    cold = np.arange(40, dtype=np.uint8).reshape(10, 4)
    assert O.gather_rows(cold, [7, 2]).tolist() == [[28, 29, 30, 31], [8, 9, 10, 11]]


def test_bias_for_fraction_counts():
    g = np.random.default_rng(11)
    z = g.standard_normal(1000) * 30
    b = O.bias_for_fraction(z, 0.1)
    assert int(((z + b) >= 0).sum()) == 100
    # the cut is the midpoint of the straddling order statistics: no entry sits on it
    zs = np.sort(z)
    assert -b == (zs[899] + zs[900]) / 2 and zs[899] < -b < zs[900]
    assert not np.any(z + b == 0)
