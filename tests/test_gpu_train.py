"""Parity of lsa_index_train_step (loss and gradients of one indexer training step) with
the fp64 oracle.  The GPU gets the oracle's bf16 c and q and its w, so both sides run the
same forward.  Gradient tolerance: 2e-3 of the sum of the absolute values of each
gradient's terms (propagated through the same chain; the key sum taken ungated, so a
sign flip of a near-zero dot product is covered), which bounds the bf16 hi/lo split of
the gated gradient (2^-17), fp32 accumulation and such flips."""
import numpy as np
import pytest
import torch

import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import build
from oracle import lsa_oracle as O
from oracle import train as T

import lsa_cases as C

pytestmark = pytest.mark.gpu
RTOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    lsa.lib()


def bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


# Head weights drawn N(0, 1/D) scaled by W_SCALE: the logits then have a spread of a few
# units (z ~ 64 * W_SCALE * 8 for H = 64, dI = 128) instead of ~64, so that nearly every
# (position, entry) pair lies inside the probability clamp |z| < ln(2^20 - 1) and the
# gradient comparison exercises the unclamped path; a few pairs still reach the clamp.
W_SCALE = 1.0 / 16
Z_CLAMP = float(np.log(2.0 ** 20 - 1))


def problem(seed, P, N, D, r, H, dI, pos=0.08, w_scale=W_SCALE):
    g = np.random.default_rng(seed)
    t = dict(h=bf16(g.standard_normal((P, D))), Wd=bf16(g.standard_normal((D, r)) / np.sqrt(D)),
             Wu=bf16(g.standard_normal((r, H * dI)) / np.sqrt(r)),
             Ww=bf16(g.standard_normal((D, H)) / np.sqrt(D) * w_scale),
             K=bf16(g.standard_normal((N, dI))))
    y = g.random((P, N)) < pos
    return {k: v.double().numpy() for k, v in t.items()}, t, y


def clamped_fraction(f, bias, H, dI, n=2048):
    """Share of (position, entry) pairs over the first n entries whose probability the
    loss clamps (zero gradient there), from the oracle's projection and score."""
    K = f["K"][:n]
    z = np.stack([O.head_fused_logits(*O.project_query(f["h"][p], f["Wd"], f["Wu"], f["Ww"], H, dI, True), bias, K)
                  for p in range(f["h"].shape[0])])
    return float((np.abs(z) > Z_CLAMP).mean())


def oracle_forward(f, H, dI):
    c = O.round_to_bf16(f["h"] @ f["Wd"])
    q = O.round_to_bf16(c @ f["Wu"])
    w = (f["h"] @ f["Ww"]).astype(np.float32).astype(np.float64)
    return c, q, w


def run_gpu(t, y, bias, gamma, H, dI, c=None, q=None, w=None):
    P, D = t["h"].shape
    r = t["Wd"].shape[1]
    N = t["K"].shape[0]
    dev = lambda x: x.cuda().contiguous()
    labels = torch.from_numpy(O.pack_bits(y).view(np.int32)).cuda()
    loss = torch.zeros(2, dtype=torch.float64, device="cuda")
    dbias = torch.zeros(1, dtype=torch.float64, device="cuda")
    dWd = torch.zeros(D, r, device="cuda")
    dWu = torch.zeros(r, H * dI, device="cuda")
    dWw = torch.zeros(D, H, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_index_train_step_workspace_bytes(P, N, D, r, H, dI))
    args = [None, None, None]
    if c is not None:
        args = [dev(bf16(c)), dev(bf16(q)), torch.from_numpy(w.astype(np.float32)).cuda()]
    lsa.lsa_index_train_step(P, N, D, r, H, dI, 1, dev(t["h"]), dev(t["Wd"]), dev(t["Wu"]), dev(t["Ww"]), bias, 1,
                             dev(t["K"]), None, labels, gamma, *args, loss, dWd, dWu, dWw, dbias, ws, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return loss.cpu().numpy(), dbias.item(), dWd.cpu().numpy(), dWu.cpu().numpy(), dWw.cpu().numpy()


def bounds(f, c, q, w, y, bias, gamma, H, dI):
    """Absolute-value propagation of every gradient's terms (ungated key sum)."""
    P = f["h"].shape[0]
    A = np.einsum("phd,sd->phs", q.reshape(P, H, dI), f["K"])
    z = np.einsum("ph,phs->ps", w, np.maximum(A, 0)) + bias
    g = np.abs(T.dloss_dz(z, y, gamma, z.size))
    Uabs = np.einsum("ps,sd->pd", g, np.abs(f["K"]))[:, None, :]
    dq = (np.abs(w)[:, :, None] * Uabs).reshape(P, H * dI)
    dw = np.einsum("phd,pd->ph", np.abs(q.reshape(P, H, dI)), Uabs[:, 0, :])
    return {"W_up": np.abs(c).T @ dq, "W_down": np.abs(f["h"]).T @ (dq @ np.abs(f["Wu"]).T),
            "W_w": np.abs(f["h"]).T @ dw, "b": float(g.sum())}


def check(got, exp_grads, bnd, exp_loss):
    loss, dbias, dWd, dWu, dWw = got
    assert loss[0] == pytest.approx(exp_loss[0], rel=1e-5) and loss[1] == pytest.approx(exp_loss[1], rel=1e-5)
    assert abs(dbias - exp_grads["b"]) <= 1e-4 * bnd["b"] + 1e-15
    for name, arr in (("W_down", dWd), ("W_up", dWu), ("W_w", dWw)):
        err = np.abs(arr - exp_grads[name])
        ok = err <= RTOL * bnd[name] + 1e-12
        assert ok.all(), f"{name}: {int((~ok).sum())} of {ok.size} outside, worst {float((err / (bnd[name] + 1e-30)).max()):.2e}"


@pytest.mark.parametrize("H,dI,P", [(64, 128, 4), (32, 64, 8), (128, 128, 3)])
def test_train_step_matches_oracle(H, dI, P):
    D, r, N, bias, gamma = 256, 64, 3001, -1.5, 2.0
    f, t, y = problem(H + dI, P, N, D, r, H, dI)
    assert clamped_fraction(f, bias, H, dI) < 0.1
    c, q, w = oracle_forward(f, H, dI)
    bce, fl, grads = T.loss_and_grads(f["h"], f["Wd"], f["Wu"], f["Ww"], bias, f["K"], y, H, dI, gamma, True)
    got = run_gpu(t, y, bias, gamma, H, dI, c, q, w)
    check(got, grads, bounds(f, c, q, w, y, bias, gamma, H, dI), (bce, fl))


def test_train_step_internal_projection_equals_given():
    """Projecting inside the call gives exactly what lsa_index_project's outputs give."""
    H, dI, P, D, r, N = 64, 128, 6, 512, 128, 2000
    f, t, y = problem(5, P, N, D, r, H, dI)
    a = run_gpu(t, y, 0.5, 2.0, H, dI)
    q = torch.empty(1, P, H, dI, dtype=torch.bfloat16, device="cuda")
    wv = torch.empty(1, P, H, device="cuda")
    ws = lsa.workspace(lsa.lsa_index_project_workspace_bytes(P, 1, D, r, H, dI, 1))
    lsa.lsa_index_project(P, 1, D, r, H, dI, 1, t["h"].cuda().reshape(1, P, D), t["Wd"].cuda().reshape(1, D, r),
                          t["Wu"].cuda().reshape(1, r, H * dI), t["Ww"].cuda().reshape(1, D, H), -1, q, wv, ws)
    torch.cuda.synchronize()
    c = O.round_to_bf16(f["h"] @ f["Wd"])          # c is not an output of the projection call
    b = run_gpu(t, y, 0.5, 2.0, H, dI, c, q.float().cpu().numpy().reshape(P, H * dI), wv.cpu().numpy().reshape(P, H))
    for x, z in zip(a[2:], b[2:]):
        assert np.abs(x - z).max() <= 1e-3 * (np.abs(z).max() + 1e-30)
    assert a[0][0] == pytest.approx(b[0][0], rel=1e-6)


def test_train_step_full_size_against_chunked_oracle():
    """P = 64 positions against N = 131,072 keys (H = 64, dI = 128, D = 4096, r = 512).
    The oracle's gradients are linear in the per-entry terms: it runs on 16 entry chunks
    (each with the full normalisation) and the chunk results are added."""
    H, dI, P, D, r, N = 64, 128, 64, 4096, 512, 131072
    f, t, y = problem(9, P, N, D, r, H, dI, pos=0.01)
    assert clamped_fraction(f, -2.0, H, dI) < 0.1
    c, q, w = oracle_forward(f, H, dI)
    got = run_gpu(t, y, -2.0, 2.0, H, dI, c, q, w)
    grads = {"W_up": 0.0, "W_down": 0.0, "W_w": 0.0, "b": 0.0}
    bnd = {"W_up": 0.0, "W_down": 0.0, "W_w": 0.0, "b": 0.0}
    bce = fl = 0.0
    nch = 16
    for i in range(nch):
        sl = slice(i * N // nch, (i + 1) * N // nch)
        fk = dict(f, K=f["K"][sl])
        scale = (sl.stop - sl.start) / N
        b_, f_, g_ = T.loss_and_grads(fk["h"], fk["Wd"], fk["Wu"], fk["Ww"], -2.0, fk["K"], y[:, sl], H, dI, 2.0, True)
        bn = bounds(fk, c, q, w, y[:, sl], -2.0, 2.0, H, dI)
        bce += b_ * scale
        fl += f_ * scale
        for k in grads:
            grads[k] = grads[k] + g_[k] * scale
            bnd[k] = bnd[k] + bn[k] * scale
    check(got, grads, bnd, (bce, fl))
