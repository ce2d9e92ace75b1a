"""Pins of the training-step oracle (CPU): central finite differences of the loss, a
closed form of dJ/dz, and the per-head weight gradient from its own definition."""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from oracle import train as T


def small_problem(seed, P=3, N=40, D=6, r=4, H=3, dI=5):
    g = np.random.default_rng(seed)
    h = g.standard_normal((P, D))
    Wd = g.standard_normal((D, r)) / np.sqrt(D)
    Wu = g.standard_normal((r, H * dI)) / np.sqrt(r)
    Ww = g.standard_normal((D, H)) / np.sqrt(D)
    K = g.standard_normal((N, dI))
    y = g.random((P, N)) < 0.3
    return h, Wd, Wu, Ww, 0.3, K, y, H, dI


def J(h, Wd, Wu, Ww, b, K, y, H, dI, gamma=2.0):
    bce, fl, _ = T.loss_and_grads(h, Wd, Wu, Ww, b, K, y, H, dI, gamma, False)
    return bce + fl


@pytest.mark.parametrize("seed", [0, 1])
def test_gradients_match_central_differences(seed):
    h, Wd, Wu, Ww, b, K, y, H, dI = small_problem(seed)
    _, _, grads = T.loss_and_grads(h, Wd, Wu, Ww, b, K, y, H, dI, 2.0, False)
    eps = 1e-6
    params = {"W_down": Wd, "W_up": Wu, "W_w": Ww}
    for name, Wt in params.items():
        for idx in np.ndindex(Wt.shape):
            Wp, Wm = Wt.copy(), Wt.copy()
            Wp[idx] += eps
            Wm[idx] -= eps
            args = lambda W: {**params, name: W}
            jp = J(h, args(Wp)["W_down"], args(Wp)["W_up"], args(Wp)["W_w"], b, K, y, H, dI)
            jm = J(h, args(Wm)["W_down"], args(Wm)["W_up"], args(Wm)["W_w"], b, K, y, H, dI)
            fd = (jp - jm) / (2 * eps)
            assert abs(fd - grads[name][idx]) <= 1e-6 + 1e-5 * abs(fd), (name, idx, fd, grads[name][idx])
    fd_b = (J(h, Wd, Wu, Ww, b + eps, K, y, H, dI) - J(h, Wd, Wu, Ww, b - eps, K, y, H, dI)) / (2 * eps)
    assert abs(fd_b - grads["b"]) <= 1e-6 + 1e-5 * abs(fd_b)


def test_dloss_dz_closed_form_at_half():
    """At z = 0 (p = 1/2), gamma = 2: y = 1 -> (1/2 - 1) + (2 * 1/2 * 1/4 * ln(1/2) - 1/8);
    y = 0 -> 1/2 + (1/8 - 2 * 1/4 * 1/2 * ln(1/2))."""
    d = T.dloss_dz(np.zeros(2), np.array([1.0, 0.0]), 2.0, 1)
    ln2 = np.log(2.0)
    assert d[0] == pytest.approx(-0.5 - ln2 / 4 - 0.125, rel=1e-14)
    assert d[1] == pytest.approx(0.5 + 0.125 + ln2 / 4, rel=1e-14)


def test_dloss_dz_zero_where_the_clamp_holds():
    """Beyond |z| = ln(2^20 - 1) ~ 13.863 the clamped probability is constant in z, so the
    loss is flat there (its central differences vanish) and dJ/dz is exactly zero, for
    either label; just inside the clamp it is not."""
    zc = np.log(2.0 ** 20 - 1)
    for z0 in (-40.0, -20.0, -14.0, 14.0, 20.0, 40.0):
        for y in (0.0, 1.0):
            z, yy = np.array([z0]), np.array([y])
            jp = sum(O.bce_focal(O.sigmoid(z + 1e-3), yy, 2.0))
            jm = sum(O.bce_focal(O.sigmoid(z - 1e-3), yy, 2.0))
            assert jp == jm, (z0, y)
            assert T.dloss_dz(z, yy, 2.0, 1)[0] == 0.0, (z0, y)
    for z0 in (-13.0, 13.0):
        assert abs(z0) < zc
        assert T.dloss_dz(np.array([z0, z0]), np.array([0.0, 1.0]), 2.0, 1).tolist().count(0.0) == 0


def test_dloss_dz_matches_differences_of_bce_focal():
    g = np.random.default_rng(3)
    z = g.standard_normal(50) * 4
    y = g.random(50) < 0.5
    eps = 1e-6
    for i in range(50):
        zp, zm = z.copy(), z.copy()
        zp[i] += eps
        zm[i] -= eps
        jp = sum(O.bce_focal(O.sigmoid(zp), y, 2.0))
        jm = sum(O.bce_focal(O.sigmoid(zm), y, 2.0))
        fd = (jp - jm) / (2 * eps)
        assert abs(fd - T.dloss_dz(z, y, 2.0, 50)[i]) <= 1e-8 + 1e-6 * abs(fd)


def test_head_weight_gradient_from_its_own_definition():
    """dw_ph computed as q_ph . U_ph equals sum_s g_ps ReLU(A_phs) written out directly."""
    h, Wd, Wu, Ww, b, K, y, H, dI = small_problem(4)
    c, q, w, A, z = T.forward(h, Wd, Wu, Ww, b, K, H, dI, False)
    g = T.dloss_dz(z, y, 2.0, z.size)
    dw_direct = np.array([[sum(g[p, s] * max(A[p, hh, s], 0.0) for s in range(K.shape[0])) for hh in range(H)]
                          for p in range(h.shape[0])])
    _, _, grads = T.loss_and_grads(h, Wd, Wu, Ww, b, K, y, H, dI, 2.0, False)
    assert np.allclose(grads["W_w"], h.T @ dw_direct, rtol=1e-12, atol=1e-15)


# ----------------------------------------------------------------------------- forward pass
#
# The backward pins above hold loss_and_grads to finite differences of a J that the same
# forward() computes, so a mistake in forward() would pass them.  The pins below hold
# forward() to the separately pinned projection and score (project_query,
# head_fused_logits, whose own pins include the hand-derived worked example), and the
# bf16 branch of the backward to finite differences of its straight-through surrogate.


def _worked():
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "score_worked_example.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("bf16", [False, True])
def test_forward_on_the_worked_example(bf16):
    """The hand-derived example (every value exact in bf16) through forward() with one
    position: c, q, w, the per-head dots and z as derived by hand."""
    ex = _worked()
    e = ex["expected"]
    h = np.array([ex["h"]], dtype=np.float64)
    c, q, w, A, z = T.forward(h, np.array(ex["W_down"], dtype=np.float64), np.array(ex["W_up"], dtype=np.float64),
                              np.array(ex["W_w"], dtype=np.float64), ex["bias"], np.array(ex["K"], dtype=np.float64),
                              ex["H"], ex["dI"], bf16)
    assert np.array_equal(c[0], e["c"])
    assert np.array_equal(q[0], e["q"])
    assert np.array_equal(w[0], e["w"])
    assert np.array_equal(A[0].T, e["dots"])      # A[p][h][s], dots[s][h]
    assert np.array_equal(z[0], e["z"])


@pytest.mark.parametrize("bf16", [False, True])
def test_forward_matches_the_pinned_projection_and_score(bf16):
    """Per position, forward()'s q and w are project_query's and its z is
    head_fused_logits' on them; the per-head dots A reproduce z through the ReLU and the
    head weights.  Random inputs, so the bf16 roundings of c and q are active."""
    h, Wd, Wu, Ww, b, K, y, H, dI = small_problem(5, P=4, N=60)
    c, q, w, A, z = T.forward(h, Wd, Wu, Ww, b, K, H, dI, bf16)
    for p in range(h.shape[0]):
        q_ref, w_ref = O.project_query(h[p], Wd, Wu, Ww, H, dI, bf16)
        if bf16:      # rounded values: equal (an fp64 sum one bit off a midpoint is ~2^-44 rare)
            assert np.array_equal(q[p], q_ref)
        else:         # batched and per-row fp64 products may differ in the last bit
            np.testing.assert_allclose(q[p], q_ref, rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(w[p], w_ref, rtol=1e-13, atol=1e-15)
        z_ref = O.head_fused_logits(q_ref, w_ref, b, K)
        np.testing.assert_allclose(z[p], z_ref, rtol=1e-13, atol=1e-13)
        for s in range(K.shape[0]):
            zs = b + sum(w_ref[hh] * max(0.0, float(q_ref[hh] @ K[s])) for hh in range(H))
            assert abs(zs - z[p, s]) <= 1e-12 * (1 + abs(zs))
            assert np.allclose(A[p, :, s], q_ref @ K[s], rtol=1e-13, atol=1e-13)
    if bf16:   # the rounding really changed something on these inputs
        q64, _ = O.project_query(h[0], Wd, Wu, Ww, H, dI, False)
        assert not np.array_equal(q[0], q64)


def test_bf16_branch_gradients_are_straight_through():
    """With bf16 boundaries the gradients are those of the straight-through surrogate:
    q(Wd', Wu') = q_r + c_r (Wu' - Wu) + (h (Wd' - Wd)) Wu', w = h Ww', where c_r and q_r
    are the rounded values at the expansion point (c_r is project_query with an identity
    up-projection, which returns the rounded c).  Finite differences of the surrogate's
    loss, evaluated through the pinned score and loss, must match the bf16 branch."""
    h, Wd, Wu, Ww, b, K, y, H, dI = small_problem(6, P=2, N=30)
    P, r = h.shape[0], Wd.shape[1]
    gamma = 2.0
    c_r = np.stack([O.project_query(h[p], Wd, np.eye(r), Ww, 1, r, True)[0][0] for p in range(P)])
    q_r = np.stack([O.project_query(h[p], Wd, Wu, Ww, H, dI, True)[0].ravel() for p in range(P)])

    def J_st(Wd2, Wu2, Ww2, b2):
        z = np.stack([O.head_fused_logits((q_r[p] + c_r[p] @ (Wu2 - Wu) + (h[p] @ (Wd2 - Wd)) @ Wu2).reshape(H, dI),
                                          h[p] @ Ww2, b2, K) for p in range(P)])
        return sum(O.bce_focal(O.sigmoid(z), y, gamma))

    bce, fl, grads = T.loss_and_grads(h, Wd, Wu, Ww, b, K, y, H, dI, gamma, True)
    assert bce + fl == pytest.approx(J_st(Wd, Wu, Ww, b), rel=1e-13)
    eps = 1e-6
    params = {"W_down": Wd, "W_up": Wu, "W_w": Ww}
    for name, Wt in params.items():
        for idx in np.ndindex(Wt.shape):
            Wp, Wm = Wt.copy(), Wt.copy()
            Wp[idx] += eps
            Wm[idx] -= eps
            a = {**params, name: Wp}
            m = {**params, name: Wm}
            fd = (J_st(a["W_down"], a["W_up"], a["W_w"], b) - J_st(m["W_down"], m["W_up"], m["W_w"], b)) / (2 * eps)
            assert abs(fd - grads[name][idx]) <= 1e-6 + 1e-5 * abs(fd), (name, idx, fd, grads[name][idx])
    fd_b = (J_st(Wd, Wu, Ww, b + eps) - J_st(Wd, Wu, Ww, b - eps)) / (2 * eps)
    assert abs(fd_b - grads["b"]) <= 1e-6 + 1e-5 * abs(fd_b)
