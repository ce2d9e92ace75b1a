"""Shared test helpers: device inputs from the seeded generator, raw copies for the
oracle, and the comparison rules (tolerance bands) used by the parity tests."""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from oracle import lsa_oracle as O
from oracle import step as OS
from synth import workloads as W

# Tolerance on I = sigmoid(z) by key dtype; on z the slope of sigmoid at 0 is 1/4.
TOL_I = {"f32": 1e-5, "bf16": 2e-3, "e4m3": 1e-2}


def tol_z(kdtype: str) -> float:
    return 4.0 * TOL_I[kdtype]


def raw(t: torch.Tensor) -> np.ndarray:
    """Device/host tensor -> numpy array of its storage (bf16 as uint16 bit patterns)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def base_name(w: W.ScoreWorkload) -> str:
    return w.name


@dataclass
class Inputs:
    w: W.ScoreWorkload
    h: torch.Tensor        # [L][B][D]
    Wd: torch.Tensor       # [L][D][r]
    Wu: torch.Tensor       # [L][r][H*dI]
    Ww: torch.Tensor       # [L][D][H]
    bias: torch.Tensor     # [L] fp32
    K: torch.Tensor        # [L][B][N][dI]
    kscale: torch.Tensor | None
    direction: torch.Tensor


def make_inputs(w: W.ScoreWorkload, device="cuda") -> Inputs:
    """Inputs of workload w (possibly reduced with W.scaled: the first B sequences and
    first N entries of the stored workload's streams)."""
    bias, direction = W.load_params(w.name)
    return make_inputs_with(w, bias[: w.L], direction[: w.B, : w.L], device)


def make_inputs_with(w: W.ScoreWorkload, bias, direction, device="cuda") -> Inputs:
    """Inputs of workload w with a given per-layer bias and planted direction."""
    h = W.hidden_states(w, device).transpose(0, 1).contiguous()
    Wd, Wu, Ww = W.all_layer_weights(w, device)
    kdt = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}[w.kdtype]
    K = torch.empty(w.L, w.B, w.N, w.dI, dtype=kdt, device=device)
    ks = torch.empty(w.L, w.B, w.N, dtype=torch.float32, device=device) if w.kdtype == "e4m3" else None
    for l in range(w.L):
        for b in range(w.B):
            k, s = W.keys(w, b, l, direction[b, l].double(), 0, w.N, device)
            K[l, b] = k
            if ks is not None:
                ks[l, b] = s
    return Inputs(w, h, Wd, Wu, Ww, bias.to(device), K, ks, direction)


class OracleCache:
    """Oracle results of (b, l) computed on demand from the raw inputs."""

    def __init__(self, inp: Inputs):
        self.inp = inp
        self.w = inp.w
        self._qw = {}
        self._h = raw(inp.h)
        self._Wd = [raw(inp.Wd[l]) for l in range(self.w.L)]
        self._Wu = [raw(inp.Wu[l]) for l in range(self.w.L)]
        self._Ww = [raw(inp.Ww[l]) for l in range(self.w.L)]

    def qw(self, l, b):
        if (l, b) not in self._qw:
            self._qw[l, b] = OS.project(self._h[l, b], self._Wd[l], self._Wu[l], self._Ww[l],
                                        self.w.H, self.w.dI, self.w.wdtype)
        return self._qw[l, b]

    def keys(self, l, b, entries=None):
        K = self.inp.K[l, b] if entries is None else self.inp.K[l, b][entries]
        s = None
        if self.inp.kscale is not None:
            s = raw(self.inp.kscale[l, b] if entries is None else self.inp.kscale[l, b][entries])
        return OS.decode_keys(raw(K), s, self.w.kdtype)

    def z(self, l, b, entries=None):
        q, wv = self.qw(l, b)
        return O.head_fused_logits(q, wv, float(raw(self.inp.bias)[l]), self.keys(l, b, entries))

    def q_allowed(self, l, b):
        """Per-element bound on |q_cuda - q_oracle| for an fp32-accumulating projection.

        The device sums in fp32 with at most FP32_DEPTH sequential additions per output,
        so |fl(sum) - sum| <= gamma * sum|terms| (gamma = depth * 2^-24 / (1 - depth * 2^-24)).
        An element of c can round to a different bf16 value than the exact sum only when
        the exact sum lies within that error of a rounding midpoint; such an element may
        move by one ulp of c.  The perturbation of the pre-rounding q is then
        (sum over those elements of ulp(c_i) |W_up[i, j]|) + gamma * sum|c_i W_up[i, j]|,
        and rounding q to bf16 adds at most one ulp of q.  For fp32 models (no rounding)
        the bound is the two fp32 summation errors alone."""
        w = self.w
        h = OS.decode(self._h[l, b], w.wdtype)
        Wd = OS.decode(self._Wd[l], w.wdtype)
        Wu = OS.decode(self._Wu[l], w.wdtype)
        u = 2.0 ** -24
        gam = FP32_DEPTH * u / (1 - FP32_DEPTH * u)
        c_exact = h @ Wd
        err_c = gam * (np.abs(h) @ np.abs(Wd))
        if w.wdtype == "bf16":
            c_r = O.round_to_bf16(c_exact)
            ulp_c = bf16_ulp(c_r)
            to_mid = np.abs(np.abs(c_exact - c_r) - ulp_c / 2)
            dc = np.where(to_mid <= err_c, ulp_c, 0.0)
        else:
            c_r, dc = c_exact, err_c
        err_q = dc @ np.abs(Wu) + gam * ((np.abs(c_r) + dc) @ np.abs(Wu))
        q, _ = self.qw(l, b)
        rnd = bf16_ulp(q) if w.wdtype == "bf16" else 0.0
        return (err_q.reshape(q.shape) + rnd) * (1 + 1e-9)

    def w_allowed(self, l, b):
        """Bound on |w_cuda - w_oracle|: one fp32 summation error."""
        w = self.w
        h = OS.decode(self._h[l, b], w.wdtype)
        Ww = OS.decode(self._Ww[l], w.wdtype)
        u = 2.0 ** -24
        return FP32_DEPTH * u / (1 - FP32_DEPTH * u) * (np.abs(h) @ np.abs(Ww))

    def z_bound_from_q(self, l, b, entries=None):
        """Bound on |z(q_cuda, w_cuda) - z(q_oracle, w_oracle)| (ReLU is 1-Lipschitz):
        sum_h |w_h| sum_d allowed_hd |k_d|  +  sum_h dw_h (ReLU(q_h.k) + sum_d allowed_hd |k_d|)."""
        q, wv = self.qw(l, b)
        Kd = self.keys(l, b, entries)
        dq = np.abs(Kd) @ self.q_allowed(l, b).T
        return dq @ np.abs(wv) + (np.maximum(Kd @ q.T, 0) + dq) @ self.w_allowed(l, b)


# Longest chain of fp32 additions behind one projected element, in units of 2^-24 relative
# error each.  CUDA cores: 256-element slices and 16 slice sums.  Tensor cores: a
# 512-element slice accumulated by tcgen05.mma, whose addition order and rounding mode
# are unspecified, counted as 512 additions of error up to 2^-23 each, then 8 fp32 slice
# sums; with margin.
FP32_DEPTH = 1100


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (2^-133 below the normal range)."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(x > 0, x, 1.0)))
    return np.where(x >= 2.0 ** -126, np.exp2(e - 7), 2.0 ** -133)


def bf16_steps_apart(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """How many bf16 values apart two bf16-valued arrays are, element by element: the
    difference of their positions on the ordered line of finite bf16 values (+0 and -0
    share position 0).  1 means adjacent values, i.e. one unit in the last place."""
    def pos(x):
        bits = (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.int64)
        return np.where(bits & 0x8000, -(bits & 0x7FFF), bits)
    assert np.array_equal(np.asarray(a, dtype=np.float32).astype(np.float64), np.asarray(a, dtype=np.float64))
    return np.abs(pos(a) - pos(b))


def assert_q_statistics(q_cuda: np.ndarray, q_oracle: np.ndarray, what=""):
    """The device's bf16 queries (any shape; pass every unit of a workload at once)
    against the oracle's: at least 97% of the elements equal and at least 99.5% within
    one bf16 step.  Neither can reach 100%, because the device sums in fp32:
    (a) an element of c whose exact value lies within the fp32 summation error of a bf16
        rounding midpoint can round to the other neighbour.  Measured on the B200: about
        one such element in a third of the (sequence, layer) units, as close as 2e-5 of
        a bf16 step to the midpoint.  The flipped element moves every q element of its
        unit by ulp(c_i) |W_up[i, j]|; that is a fraction of q's own spacing for most,
        but up to hundreds of steps for elements near zero, and it left 85% of one unit
        exact;
    (b) a q element whose exact value is far below its terms (cancellation) carries an
        fp32 error larger than its own bf16 spacing.
    Measured share equal / within one step: 128K 99.66% / 99.97%, 512K 98.31% / 99.73%,
    1M 99.66% / 99.95%.  Every element stays inside the rigorous bound q_allowed, and the
    scoring is held to the oracle through the oracle's own query."""
    steps = bf16_steps_apart(q_cuda, q_oracle)
    exact = float((steps == 0).mean())
    within1 = float((steps <= 1).mean())
    assert exact >= 0.97, f"{what}: only {exact:.5f} of the query elements equal the oracle's"
    assert within1 >= 0.995, f"{what}: only {within1:.5f} of the query elements within one bf16 step"
    return exact, within1


def q_within(q_cuda: np.ndarray, q_oracle: np.ndarray, allowed: np.ndarray) -> np.ndarray:
    return np.abs(q_cuda - q_oracle) <= allowed


def unpack(words: torch.Tensor, n: int) -> np.ndarray:
    return O.unpack_bits(raw(words).view(np.uint32), n)


def band(z_oracle: np.ndarray, tz) -> np.ndarray:
    """Entries whose oracle logit lies within the tolerance of the threshold."""
    return np.abs(z_oracle) <= tz


def assert_mask_parity(got: np.ndarray, z_oracle: np.ndarray, tz, what=""):
    exp = O.threshold_mark(z_oracle)
    bad = (got != exp) & ~band(z_oracle, tz)
    assert not bad.any(), f"{what}: {int(bad.sum())} mask mismatches outside the band, e.g. {np.flatnonzero(bad)[:5]}"


def sigmoid_tol_ok(score: np.ndarray, z_oracle: np.ndarray, tol_I) -> np.ndarray:
    return np.abs(score - O.sigmoid(z_oracle)) <= tol_I
