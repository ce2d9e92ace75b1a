"""Strength of the oracle's pins.  Each plausible mistake below is planted in the oracle
(on the CPU, through monkeypatch, for the duration of one case) and at least one pin test
must then fail.  A mistake that every pin survives could reach the parity tests unnoticed,
since those trust the oracle.

The pins are the tests of tests/test_oracle_pins.py, tests/test_oracle_train.py and
tests/test_oracle_hot_pool.py, run as plain functions (parametrized cases expanded)."""
from __future__ import annotations

import importlib.util
import os

import numpy as np
import pytest

from oracle import lsa_oracle as O
from oracle import train as T

HERE = os.path.dirname(os.path.abspath(__file__))
PIN_MODULES = ("test_oracle_pins", "test_oracle_train", "test_oracle_hot_pool")


def _load(name):
    spec = importlib.util.spec_from_file_location(f"_pins_{name}", os.path.join(HERE, name + ".py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _pin_calls():
    """(label, zero-argument callable) for every pin test."""
    calls = []
    for mod_name in PIN_MODULES:
        mod = _load(mod_name)
        for name, f in vars(mod).items():
            if not (name.startswith("test_") and callable(f)):
                continue
            marks = [m for m in getattr(f, "pytestmark", []) if m.name == "parametrize"]
            if not marks:
                calls.append((f"{mod_name}.{name}", f))
                continue
            assert len(marks) == 1, name
            argnames, values = marks[0].args[0], marks[0].args[1]
            names = [a.strip() for a in argnames.split(",")]
            for v in values:
                vals = tuple(v) if len(names) > 1 else (v,)
                calls.append((f"{mod_name}.{name}{list(vals)}",
                              lambda f=f, kw=dict(zip(names, vals)): f(**kw)))
    return calls


PINS = _pin_calls()


def _first_failing_pin():
    for label, call in PINS:
        try:
            call()
        except Exception:               # an assertion, or an error the mistake provokes
            return label
    return None


def test_pins_pass_on_the_oracle_as_it_stands():
    assert len(PINS) >= 30
    assert _first_failing_pin() is None


# ----------------------------------------------------------------------------- mistakes


def score_without_relu(q, w, b, K):
    K = np.asarray(K, dtype=np.float64)
    return (K @ np.asarray(q, dtype=np.float64).T) @ np.asarray(w, dtype=np.float64) + b


def score_without_bias(q, w, b, K):
    K = np.asarray(K, dtype=np.float64)
    return np.maximum(K @ np.asarray(q, dtype=np.float64).T, 0.0) @ np.asarray(w, dtype=np.float64)


def score_weight_inside_relu(q, w, b, K):
    K = np.asarray(K, dtype=np.float64)
    dots = K @ np.asarray(q, dtype=np.float64).T
    return np.maximum(dots * np.asarray(w, dtype=np.float64), 0.0).sum(axis=1) + b


def score_transposed_query(q, w, b, K):
    q = np.asarray(q, dtype=np.float64)
    H, dI = q.shape
    qt = q.reshape(dI, H).T                 # reading [H][dI] as if it were [dI][H]
    return np.maximum(np.asarray(K, dtype=np.float64) @ qt.T, 0.0) @ np.asarray(w, dtype=np.float64) + b


def threshold_strict(z):
    return np.asarray(z) > 0.0


def project_without_c_rounding(h, W_down, W_up, W_w, H, dI, bf16_boundaries):
    h = np.asarray(h, dtype=np.float64)
    c = h @ np.asarray(W_down, dtype=np.float64)
    q = c @ np.asarray(W_up, dtype=np.float64)
    if bf16_boundaries:
        q = O.round_to_bf16(q)
    return q.reshape(H, dI), h @ np.asarray(W_w, dtype=np.float64)


_round_to_bf16 = O.round_to_bf16


def round_ties_away(x):
    x = np.asarray(x, dtype=np.float64)
    out = _round_to_bf16(x)
    fin = np.isfinite(x) & (x != 0)
    m, e = np.frexp(x[fin])
    e_q = np.maximum(e, -125)
    s = np.ldexp(m, 8 + e - e_q)
    away = np.ldexp(np.sign(s) * np.floor(np.abs(s) + 0.5), e_q - 8)
    out[fin] = away
    return out


_decode_e4m3 = O.decode_e4m3


def e4m3_exponent_off_by_one(u8):
    return _decode_e4m3(u8) * 2.0


def union_against_final(marks_by_layer):
    ms = [np.asarray(m, dtype=bool) for m in marks_by_layer]
    U = np.zeros_like(ms[0])
    for m in ms:
        U = U | m
    return U, [m & ~U for m in ms]


def compact_descending(mark):
    return np.flatnonzero(np.asarray(mark, dtype=bool))[::-1].astype(np.int64)


def topk_ties_high_index(fetched_idx, key_of_entry, k):
    idx = np.asarray(fetched_idx, dtype=np.int64)
    if idx.size == 0 or k <= 0:
        return np.zeros(0, dtype=np.int64)
    key = np.asarray(key_of_entry, dtype=np.float64)[idx]
    order = np.lexsort((-idx, -key))
    return np.sort(idx[order[:k]])


def topk_rank_order(fetched_idx, key_of_entry, k):
    idx = np.asarray(fetched_idx, dtype=np.int64)
    if idx.size == 0 or k <= 0:
        return np.zeros(0, dtype=np.int64)
    key = np.asarray(key_of_entry, dtype=np.float64)[idx]
    return idx[np.lexsort((idx, -key))[:k]]


def fetched_key_all_layers(z_by_layer, marks_by_layer):
    return np.asarray(z_by_layer, dtype=np.float64).max(axis=0)


def _nucleus(x, top_p, strict_after=False, ties_high=False, inclusive=False):
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(x - x.max())
    pi = e / e.sum()
    n = np.arange(x.size)
    order = np.lexsort((-n if ties_high else n, -pi))
    cum = np.cumsum(pi[order])
    before = cum - pi[order]
    sel = np.zeros(x.size, dtype=bool)
    if strict_after:
        sel[order] = cum < top_p          # drops the entry that crosses top_p
    elif inclusive:
        sel[order] = before <= top_p
    else:
        sel[order] = before < top_p
    return sel


def vote_strict_count(logits, top_p, theta):
    x = np.asarray(logits)
    L, P, N = x.shape
    count = np.zeros((P, N), dtype=np.int64)
    for l in range(L):
        for p in range(P):
            count[p] += O.nucleus(x[l, p], top_p)
    return count > theta, count


def bce_focal_gamma_minus_one(prob, label, gamma, eps=O.PROB_EPS):
    return _bce_focal(prob, label, gamma - 1.0, eps)


def bce_focal_swapped_logs(prob, label, gamma, eps=O.PROB_EPS):
    return _bce_focal(1.0 - np.asarray(prob, dtype=np.float64), label, gamma, eps)


def bce_focal_no_clamp(prob, label, gamma, eps=O.PROB_EPS):
    return _bce_focal(prob, label, gamma, 0.0)


_bce_focal = O.bce_focal


def bias_without_midpoint(z_pre, frac):
    z = np.sort(np.asarray(z_pre, dtype=np.float64).ravel())
    n = z.size
    m = min(max(int(round(frac * n)), 1), n - 1)
    return float(-z[n - m])                 # puts the cut exactly on an order statistic


_dloss_dz = T.dloss_dz


def dloss_without_focal(z, y, gamma, n, eps=O.PROB_EPS):
    z = np.asarray(z, dtype=np.float64)
    p = O.sigmoid(z)
    clamped = (p < eps) | (p > 1.0 - eps)
    return np.where(clamped, 0.0, np.clip(p, eps, 1.0 - eps) - np.asarray(y, dtype=np.float64)) / n


def dloss_ignores_clamp(z, y, gamma, n, eps=O.PROB_EPS):
    z = np.asarray(z, dtype=np.float64)
    return _dloss_dz(z, y, gamma, n, eps=0.0)


def grads_without_relu_gate(h, Wd, Wu, Ww, b, K, y, H, dI, gamma, bf16_boundaries):
    h = np.asarray(h, dtype=np.float64)
    c, q, w, A, z = T.forward(h, Wd, Wu, Ww, b, K, H, dI, bf16_boundaries)
    P, N = z.shape
    bce, fl = O.bce_focal(O.sigmoid(z), y, gamma)
    g = T.dloss_dz(z, y, gamma, P * N)
    U = np.einsum("ps,sd->pd", g, K)[:, None, :].repeat(H, axis=1)      # the 1[A > 0] factor dropped
    dq = w[:, :, None] * U
    dw = np.einsum("phd,phd->ph", q, U)
    dq2 = dq.reshape(P, H * dI)
    return bce, fl, {"W_up": c.T @ dq2, "W_down": h.T @ (dq2 @ Wu.T), "W_w": h.T @ dw, "b": float(g.sum())}


_hot_update = O.HotPool.update


def hot_pool_pairs_in_age_order(self, U, t, cold=None, hot=None):
    """Moves paired with the taken slots in (stamp, slot) order, not ascending slot order."""
    U = sorted(set(int(e) for e in U))
    kept = set()
    for e in U:
        s = self.slot_of[e]
        if s >= 0:
            self.stamp[s] = t
            kept.add(s)
    need = [e for e in U if self.slot_of[e] < 0]
    if len(U) > self.slots:
        return None
    cand = sorted((self.stamp[s], s) for s in range(self.slots) if s not in kept)
    taken = [s for _, s in cand[: len(need)]]
    moves = []
    for e, s in zip(need, taken):
        old = self.entry_of[s]
        if old >= 0:
            self.slot_of[old] = -1
        self.entry_of[s], self.slot_of[e], self.stamp[s] = e, s, t
        if cold is not None:
            hot[s] = cold[e]
        moves.append((e, s))
    return moves


def hot_pool_keeps_old_stamps(self, U, t, cold=None, hot=None):
    """Resident entries of the fetch set keep their old stamps (no refresh on a hit)."""
    saved = list(self.stamp)
    keep = {self.slot_of[int(e)] for e in U if self.slot_of[int(e)] >= 0}
    moves = _hot_update(self, U, t, cold, hot)
    for s in keep:
        self.stamp[s] = saved[s]
    return moves


def sigmoid_wrong_sign(z):
    return 1.0 / (1.0 + np.exp(np.asarray(z, dtype=np.float64)))


_unpack_bits = O.unpack_bits


def unpack_shifted(words, n):
    return np.roll(_unpack_bits(words, n), 1, axis=-1)


def score_scaled(q, w, b, K):
    q = np.asarray(q, dtype=np.float64)
    dots = np.asarray(K, dtype=np.float64) @ q.T / np.sqrt(q.shape[1])
    return np.maximum(dots, 0.0) @ np.asarray(w, dtype=np.float64) + b


def nucleus_on_raw_logits(x, top_p):
    """Mass taken from the logits shifted to be positive instead of from the softmax."""
    x = np.asarray(x, dtype=np.float64)
    v = x - x.min() + 1.0
    pi = v / v.sum()
    order = np.lexsort((np.arange(x.size), -pi))
    before = np.cumsum(pi[order]) - pi[order]
    sel = np.zeros(x.size, dtype=bool)
    sel[order] = before < top_p
    return sel


def topk_padded(fetched_idx, key_of_entry, k):
    out = _topk(fetched_idx, key_of_entry, k)
    if 0 < out.size < k:
        out = np.sort(np.concatenate([out, np.full(k - out.size, out[-1])]))
    return out


_topk = O.topk_in_fetched


def hot_pool_evicts_most_recent(self, U, t, cold=None, hot=None):
    U = sorted(set(int(e) for e in U))
    kept = set()
    for e in U:
        s = self.slot_of[e]
        if s >= 0:
            self.stamp[s] = t
            kept.add(s)
    need = [e for e in U if self.slot_of[e] < 0]
    if len(U) > self.slots:
        return None
    cand = sorted(((-self.stamp[s] if self.stamp[s] else -10 ** 9), s) for s in range(self.slots) if s not in kept)
    taken = sorted(s for _, s in cand[: len(need)])
    moves = []
    for e, s in zip(need, taken):
        old = self.entry_of[s]
        if old >= 0:
            self.slot_of[old] = -1
        self.entry_of[s], self.slot_of[e], self.stamp[s] = e, s, t
        if cold is not None:
            hot[s] = cold[e]
        moves.append((e, s))
    return moves


def hot_pool_moved_rows_unstamped(self, U, t, cold=None, hot=None):
    moves = _hot_update(self, U, t, cold, hot)
    for _, s in moves or []:
        self.stamp[s] = 0
    return moves


def hot_pool_capacity_on_need(self, U, t, cold=None, hot=None):
    U = sorted(set(int(e) for e in U))
    need = [e for e in U if self.slot_of[e] < 0]
    if len(need) > self.slots:
        return None
    if len(U) > self.slots:            # fits by the (wrong) count of missing rows: move what fits
        U = [e for e in U if self.slot_of[e] >= 0] + need[: self.slots - sum(self.slot_of[e] >= 0 for e in U)]
    return _hot_update(self, U, t, cold, hot)


from oracle import step as OS  # noqa: E402  (the step-level mistakes below patch it)

_select = OS.select


def step_topk_over_last_new_set(marks_by_layer, z_by_layer, k):
    out = _select(marks_by_layer, z_by_layer, k)
    out["topk"] = O.topk_in_fetched(out["idx_new"][-1], out["key"], k)
    return out


def step_scale_ignored(K_raw, kscale, kdtype):
    return OS.decode(K_raw, kdtype)


def step_scale_divides(K_raw, kscale, kdtype):
    K = OS.decode(K_raw, kdtype)
    if kdtype == "e4m3":
        K = K / np.asarray(kscale, dtype=np.float32).astype(np.float64)[:, None]
    return K


def step_projection_without_bf16_boundaries(h_raw, Wd_raw, Wu_raw, Ww_raw, H, dI, wdtype):
    return O.project_query(OS.decode(h_raw, wdtype), OS.decode(Wd_raw, wdtype), OS.decode(Wu_raw, wdtype),
                           OS.decode(Ww_raw, wdtype), H, dI, bf16_boundaries=False)



def _forward_variant(relu=True, bias=True, round_c=True, round_q=True, w_from="h", round_w=False,
                     weight_inside=False):
    def forward(h, Wd, Wu, Ww, b, K, H, dI, bf16_boundaries):
        c = h @ Wd
        if bf16_boundaries and round_c:
            c = O.round_to_bf16(c)
        q = c @ Wu
        if bf16_boundaries and round_q:
            q = O.round_to_bf16(q)
        q = q.reshape(h.shape[0], H, dI)
        w = h @ Ww if w_from == "h" else c @ Ww[: c.shape[1]]
        if round_w:
            w = O.round_to_bf16(w)
        A = np.einsum("phd,sd->phs", q, K)
        if weight_inside:
            z = np.maximum(np.einsum("ph,phs->ps", w, A), 0.0)
        else:
            z = np.einsum("ph,phs->ps", w, np.maximum(A, 0.0) if relu else A)
        return c, q, w, A, z + (b if bias else 0.0)
    return forward


def grads_bf16_backward_with_unrounded_c(h, Wd, Wu, Ww, b, K, y, H, dI, gamma, bf16_boundaries):
    bce, fl, grads = _orig_loss_and_grads(h, Wd, Wu, Ww, b, K, y, H, dI, gamma, bf16_boundaries)
    h = np.asarray(h, dtype=np.float64)
    _, q, w, A, z = T.forward(h, Wd, Wu, Ww, b, K, H, dI, bf16_boundaries)
    g = T.dloss_dz(z, y, gamma, z.size)
    U = np.einsum("ps,phs,sd->phd", g, (A > 0).astype(np.float64), K)
    dq = (w[:, :, None] * U).reshape(h.shape[0], H * dI)
    return bce, fl, {**grads, "W_up": (h @ Wd).T @ dq}     # c before its rounding


_orig_loss_and_grads = T.loss_and_grads



def fine_scores_with_bias(q_f, w_f, K_f, fetched_idx):
    return O.head_fused_logits(q_f, w_f, 1.0, np.asarray(K_f, dtype=np.float64)[np.asarray(fetched_idx, dtype=np.int64)])


def fine_scores_without_relu(q_f, w_f, K_f, fetched_idx):
    K = np.asarray(K_f, dtype=np.float64)[np.asarray(fetched_idx, dtype=np.int64)]
    return (K @ np.asarray(q_f, dtype=np.float64).T) @ np.asarray(w_f, dtype=np.float64)


def fine_topk_over_all_entries(q_f, w_f, K_f, fetched_idx, k):
    allidx = np.arange(np.asarray(K_f).shape[0])
    key = O.fine_index_scores(q_f, w_f, K_f, allidx)
    return O.topk_in_fetched(allidx, key, k)


MISTAKES = {
    "step top-k over the last layer's new set": (OS, "select", step_topk_over_last_new_set),
    "step e4m3 scale ignored": (OS, "decode_keys", step_scale_ignored),
    "step e4m3 scale divides": (OS, "decode_keys", step_scale_divides),
    "step projection without bf16 boundaries": (OS, "project", step_projection_without_bf16_boundaries),
    "sigmoid with the wrong sign": (O, "sigmoid", sigmoid_wrong_sign),
    "bit unpacking shifted by one": (O, "unpack_bits", unpack_shifted),
    "score scaled by 1/sqrt(dI)": (O, "head_fused_logits", score_scaled),
    "nucleus mass from raw logits": (O, "nucleus", nucleus_on_raw_logits),
    "top-k padded to k": (O, "topk_in_fetched", topk_padded),
    "hot pool evicts the most recent": (O.HotPool, "update", hot_pool_evicts_most_recent),
    "hot pool moved rows unstamped": (O.HotPool, "update", hot_pool_moved_rows_unstamped),
    "hot pool capacity on missing rows": (O.HotPool, "update", hot_pool_capacity_on_need),
    "score without the ReLU": (O, "head_fused_logits", score_without_relu),
    "score without the bias": (O, "head_fused_logits", score_without_bias),
    "head weight inside the ReLU": (O, "head_fused_logits", score_weight_inside_relu),
    "query read transposed": (O, "head_fused_logits", score_transposed_query),
    "threshold I > 0.5": (O, "threshold_mark", threshold_strict),
    "c not rounded to bf16": (O, "project_query", project_without_c_rounding),
    "bf16 ties away from zero": (O, "round_to_bf16", round_ties_away),
    "e4m3 exponent off by one": (O, "decode_e4m3", e4m3_exponent_off_by_one),
    "new-sets against the final union": (O, "or_union", union_against_final),
    "fetch list descending": (O, "compact", compact_descending),
    "top-k ties to the higher index": (O, "topk_in_fetched", topk_ties_high_index),
    "top-k in rank order": (O, "topk_in_fetched", topk_rank_order),
    "top-k key over unmarked layers": (O, "fetched_key", fetched_key_all_layers),
    "nucleus drops the crossing entry": (O, "nucleus", lambda x, p: _nucleus(x, p, strict_after=True)),
    "nucleus ties to the higher index": (O, "nucleus", lambda x, p: _nucleus(x, p, ties_high=True)),
    "nucleus keeps mass-before == top_p": (O, "nucleus", lambda x, p: _nucleus(x, p, inclusive=True)),
    "vote count > theta": (O, "vote_labels", vote_strict_count),
    "focal exponent gamma - 1": (O, "bce_focal", bce_focal_gamma_minus_one),
    "BCE logs swapped": (O, "bce_focal", bce_focal_swapped_logs),
    "probabilities not clamped": (O, "bce_focal", bce_focal_no_clamp),
    "bias on an order statistic": (O, "bias_for_fraction", bias_without_midpoint),
    "dJ/dz without the focal part": (T, "dloss_dz", dloss_without_focal),
    "dJ/dz ignores the clamp": (T, "dloss_dz", dloss_ignores_clamp),
    "backward without the ReLU gate": (T, "loss_and_grads", grads_without_relu_gate),
    "hot pool pairs in age order": (O.HotPool, "update", hot_pool_pairs_in_age_order),
    "hot pool hit keeps the old stamp": (O.HotPool, "update", hot_pool_keeps_old_stamps),
    "fine score with a bias": (O, "fine_index_scores", fine_scores_with_bias),
    "fine score without the ReLU": (O, "fine_index_scores", fine_scores_without_relu),
    "fine top-k over all entries": (O, "fine_topk", fine_topk_over_all_entries),
    "training forward without the ReLU": (T, "forward", _forward_variant(relu=False)),
    "training forward drops the bias": (T, "forward", _forward_variant(bias=False)),
    "training forward with c not rounded": (T, "forward", _forward_variant(round_c=False)),
    "training forward with q not rounded": (T, "forward", _forward_variant(round_q=False)),
    "training forward with w from c": (T, "forward", _forward_variant(w_from="c")),
    "training forward with w rounded to bf16": (T, "forward", _forward_variant(round_w=True)),
    "training forward with the head weight inside the ReLU": (T, "forward", _forward_variant(weight_inside=True)),
    "training bf16 backward with unrounded c": (T, "loss_and_grads", grads_bf16_backward_with_unrounded_c),
}


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_planted_mistake_fails_a_pin(name, monkeypatch):
    target, attr, wrong = MISTAKES[name]
    monkeypatch.setattr(target, attr, wrong)
    assert _first_failing_pin() is not None, f"no pin catches: {name}"
