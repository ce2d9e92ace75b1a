"""Loss and gradients of one indexer training step, in fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle.lsa_oracle``): only the tests, the smoke check
and the benchmark's CPU baseline use it.

[SUMMARY] §2.3 (backbone-free decoupled training): the compressed indexer keys K_IComp
are precomputed and frozen; only the query side is trained; the objective is binary
cross-entropy combined with a focal loss that down-weights easy negatives.  §2.2: the
labels are the cross-layer majority-vote golden bits.

Readings (the pages give the ingredients, not the formulas):
  * one step covers one indexer layer and P query positions (hidden states h_p) scored
    against the same N frozen keys; labels y[p][s] in {0, 1};
  * objective J = BCE + FL, the two means over all P*N (p, s) pairs (as in
    ``lsa_oracle.bce_focal``), with probabilities clamped to [eps, 1 - eps]: where the
    clamp is active the derivative is zero;
  * trainable: W_down, W_up, W_w and the layer bias b;
  * the bf16 roundings of c and q in the forward pass (bf16 models) pass gradients
    through unchanged (straight-through); the gradients are computed in fp64.
"""
from __future__ import annotations

import numpy as np

from . import lsa_oracle as O


def dloss_dz(z, y, gamma: float, n: int, eps: float = O.PROB_EPS) -> np.ndarray:
    """d(BCE + FL)/dz per (p, s) for J averaged over n pairs; p = sigmoid(z).

    d BCE/dz = p - y.
    FL, y = 1: -(1-p)^g ln p      -> d/dz = g p (1-p)^g ln p - (1-p)^(g+1)
    FL, y = 0: -p^g ln(1-p)       -> d/dz = p^(g+1) - g p^g (1-p) ln(1-p)
    (dp/dz = p (1-p)); zero where the clamp is active."""
    z = np.asarray(z, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    p = O.sigmoid(z)
    clamped = (p < eps) | (p > 1.0 - eps)
    pc = np.clip(p, eps, 1.0 - eps)
    g = gamma
    d_bce = pc - y
    d_fl_pos = g * pc * (1 - pc) ** g * np.log(pc) - (1 - pc) ** (g + 1)
    d_fl_neg = pc ** (g + 1) - g * pc ** g * (1 - pc) * np.log1p(-pc)
    d = d_bce + np.where(y > 0, d_fl_pos, d_fl_neg)
    return np.where(clamped, 0.0, d) / n


def forward(h, Wd, Wu, Ww, b: float, K, H: int, dI: int, bf16_boundaries: bool):
    """(c [P][r], q [P][H][dI], w [P][H], A [P][H][N], z [P][N]) from fp64 inputs."""
    c = h @ Wd
    if bf16_boundaries:
        c = O.round_to_bf16(c)
    q = c @ Wu
    if bf16_boundaries:
        q = O.round_to_bf16(q)
    q = q.reshape(h.shape[0], H, dI)
    w = h @ Ww
    A = np.einsum("phd,sd->phs", q, K)
    z = np.einsum("ph,phs->ps", w, np.maximum(A, 0.0)) + b
    return c, q, w, A, z


def loss_and_grads(h, Wd, Wu, Ww, b: float, K, y, H: int, dI: int, gamma: float, bf16_boundaries: bool):
    """(bce, fl, grads) with grads = dict(W_down, W_up, W_w, b) of J = bce + fl.

    Backward, from z_ps = sum_h w_ph ReLU(A_phs) + b, A_phs = q_ph . k_s:
      g_ps   = dJ/dz_ps                       (dloss_dz)
      U_ph   = sum_s g_ps 1[A_phs > 0] k_s    ([P][H][dI])
      dq_ph  = w_ph U_ph;   dw_ph = q_ph . U_ph  (= sum_s g_ps ReLU(A_phs));   db = sum g
      dW_up  = c^T dq;  dc = dq W_up^T;  dW_down = h^T dc;  dW_w = h^T dw."""
    h = np.asarray(h, dtype=np.float64)
    c, q, w, A, z = forward(h, Wd, Wu, Ww, b, K, H, dI, bf16_boundaries)
    P, N = z.shape
    bce, fl = O.bce_focal(O.sigmoid(z), y, gamma)
    g = dloss_dz(z, y, gamma, P * N)
    U = np.einsum("ps,phs,sd->phd", g, (A > 0).astype(np.float64), K)
    dq = w[:, :, None] * U
    dw = np.einsum("phd,phd->ph", q, U)
    dq2 = dq.reshape(P, H * dI)
    grads = {
        "W_up": c.T @ dq2,
        "W_down": h.T @ (dq2 @ Wu.T),
        "W_w": h.T @ dw,
        "b": float(g.sum()),
    }
    return bce, fl, grads
