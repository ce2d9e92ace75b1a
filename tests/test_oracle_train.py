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
