"""Seeded synthetic inputs shaped like the workloads of Lookahead Sparse Attention.

The pages describe the indexer on DeepSeek-V4-Flash with 4:1-compressed CSA entries,
16K-512K training contexts and 1M-token serving (technical summary of
FlashMemory-DeepSeek-V4 on gist.science, §2.1 and §2.3; the podcast page's summary
for 1M).  No dataset or trained weight is used: every tensor below is drawn from the
counter-based generator in ``synth.rng``, so the oracle and the CUDA path read the
same bytes.

Recipe (identical for every workload of the scoring step):
  * h ~ N(0, 1) per (sequence, indexer layer, hidden unit).
  * W_down ~ N(0, 1/D), W_up ~ N(0, 1/r), W_w ~ N(0, 1/D), one set per indexer layer.
  * K_IComp ~ N(0, 1), except a seeded planted set of entries (the same entries in
    every layer of a sequence) drawn as k = 2 * u + N(0, 0.5) (0.5 is the variance),
    where u is a unit direction supplied by the caller; the stored workload
    parameters hold u = unit(mean over heads of q) for each (sequence, layer).
  * bf16 keys: the fp64 draw rounded to fp32 then to bf16 (round to nearest even).
  * e4m3 keys: per-entry scale s = fp32(max_d |k_d| / 448), code = e4m3(k / s)
    rounded to nearest even with saturation to +-448.
  * cold-pool rows: seeded pseudo-random 32-bit words (the gather is a byte copy).
  * vote logits: N(0, 1); per query position a seeded 1% of entries is boosted by +6
    in a seeded random 3-8 of the L layers.

Nothing here computes a query, a score, a mask or a label.
"""
from __future__ import annotations

import base64
import json
import math
import os
from dataclasses import dataclass, field

import torch

from . import rng

# Stream identifiers (any fixed small integers will do; they only separate streams).
_S_H, _S_WDOWN, _S_WUP, _S_WW, _S_FRAC, _S_PLANT, _S_KNOISE, _S_COLD = range(1, 9)
_S_VOTE_X, _S_VOTE_BOOST_SET, _S_VOTE_BOOST_LAYERS, _S_VOTE_NLAYERS, _S_POS_H = range(20, 25)
_S_DRIFT = 30
_S_FINE_Q, _S_FINE_W = 40, 41

E4M3_MAX = 448.0

_HERE = os.path.dirname(os.path.abspath(__file__))
PARAMS_PATH = os.path.join(os.path.dirname(_HERE), "tests", "golden", "workload_params.json")


@dataclass(frozen=True)
class ScoreWorkload:
    """One configuration of the scoring + selection step."""
    name: str
    B: int            # sequences
    L: int            # indexer layers (the pages place them at layers 10, 12 and 20)
    D: int            # hidden size
    r: int            # low-rank query dimension
    H: int            # indexer heads H_I
    dI: int           # indexer head dimension d_I
    N: int            # compressed entries per sequence (4:1 CSA)
    k: int            # top-k inside the fetched set
    kdtype: str       # "f32" | "bf16" | "e4m3"
    wdtype: str       # "f32" | "bf16" (h and weights)
    row_bytes: int    # bytes of one compressed-KV row in the cold pool
    plant_lo: float   # planted fraction range per sequence
    plant_hi: float
    seed: int
    layer_ids: tuple = (10, 12, 20)

    @property
    def entries(self) -> int:
        return self.B * self.L * self.N


@dataclass(frozen=True)
class VoteWorkload:
    name: str
    L: int
    P: int
    N: int
    boost: float
    boost_frac: float
    min_layers: int
    max_layers: int
    top_p: float
    theta: int
    gamma: float
    seed: int
    score_source: str = "lsa_step_512k_b8_bf16"


WORKLOADS = {
    # 16K tokens at 4:1 compression, fp32 everywhere; small enough for the oracle.
    "lsa_step_16k_tiny_fp32": ScoreWorkload(
        "lsa_step_16k_tiny_fp32", B=1, L=1, D=512, r=64, H=8, dI=64, N=4096, k=64,
        kdtype="f32", wdtype="f32", row_bytes=576 * 4, plant_lo=0.08, plant_hi=0.08,
        seed=0, layer_ids=(10,)),
    # DeepSeek-V4-Flash-shaped indexer, one 128K-token sequence.
    "lsa_step_128k_b1_bf16": ScoreWorkload(
        "lsa_step_128k_b1_bf16", B=1, L=3, D=4096, r=512, H=64, dI=128, N=32768, k=512,
        kdtype="bf16", wdtype="bf16", row_bytes=576 * 2, plant_lo=0.08, plant_hi=0.08,
        seed=1),
    # 512K-token decode batch of 8 sequences.
    "lsa_step_512k_b8_bf16": ScoreWorkload(
        "lsa_step_512k_b8_bf16", B=8, L=3, D=4096, r=512, H=64, dI=128, N=131072, k=512,
        kdtype="bf16", wdtype="bf16", row_bytes=576 * 2, plant_lo=0.02, plant_hi=0.15,
        seed=2),
    # 1M-token decode batch of 32 sequences, fp8 e4m3 keys with a per-entry fp32 scale.
    "lsa_step_1m_b32_fp8": ScoreWorkload(
        "lsa_step_1m_b32_fp8", B=32, L=3, D=4096, r=512, H=64, dI=128, N=262144, k=2048,
        kdtype="e4m3", wdtype="bf16", row_bytes=576 * 2, plant_lo=0.02, plant_hi=0.15,
        seed=3),
}

VOTE_WORKLOADS = {
    "vote_labels_l24_p64_n131072": VoteWorkload(
        "vote_labels_l24_p64_n131072", L=24, P=64, N=131072, boost=6.0, boost_frac=0.01,
        min_layers=3, max_layers=8, top_p=0.6, theta=3, gamma=2.0, seed=4),
}


def scaled(w: ScoreWorkload, **kw) -> ScoreWorkload:
    """A copy of a workload with some sizes replaced (for reduced-size test cases)."""
    d = dict(w.__dict__)
    d.update(kw)
    return ScoreWorkload(**d)


def _torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _to_storage(x64: torch.Tensor, dtype: str) -> torch.Tensor:
    """fp64 draw -> fp32 (nearest even) -> storage dtype (nearest even)."""
    x32 = x64.to(torch.float32)
    return x32 if dtype == "f32" else x32.to(torch.bfloat16)


# ----------------------------------------------------------------------------- weights

def hidden_states(w: ScoreWorkload, device="cpu") -> torch.Tensor:
    """h [B][L][D] in w.wdtype."""
    out = torch.empty(w.B, w.L, w.D, dtype=_torch_dtype(w.wdtype), device=device)
    for b in range(w.B):
        for l in range(w.L):
            key = rng.stream_key(w.seed, _S_H, b, l)
            out[b, l] = _to_storage(rng.normal(key, rng.arange(w.D, device=device)), w.wdtype)
    return out


def drifted_hidden_states(w: ScoreWorkload, t: int, rho: float, device="cpu") -> torch.Tensor:
    """h [B][L][D] at trigger t >= 1 of a sequence of triggers whose hidden states follow
    an AR(1) walk: h_1 = hidden_states(w), h_t = rho h_{t-1} + sqrt(1 - rho^2) eps_t with
    eps_t ~ N(0, 1) from its own stream (fp64, stored in w.wdtype)."""
    h = torch.empty(w.B, w.L, w.D, dtype=torch.float64, device=device)
    for b in range(w.B):
        for l in range(w.L):
            h[b, l] = rng.normal(rng.stream_key(w.seed, _S_H, b, l), rng.arange(w.D, device=device))
    c = math.sqrt(max(0.0, 1.0 - rho * rho))
    for step in range(2, t + 1):
        for b in range(w.B):
            for l in range(w.L):
                eps = rng.normal(rng.stream_key(w.seed, _S_DRIFT, b, l, step), rng.arange(w.D, device=device))
                h[b, l] = rho * h[b, l] + c * eps
    return _to_storage(h, w.wdtype)


def layer_weights(w: ScoreWorkload, l: int, device="cpu"):
    """(W_down [D][r], W_up [r][H*dI], W_w [D][H]) of indexer layer l, in w.wdtype."""
    def draw(stream, rows, cols, fan_in):
        key = rng.stream_key(w.seed, stream, l)
        x = rng.normal(key, rng.arange(rows * cols, device=device)) * (1.0 / math.sqrt(fan_in))
        return _to_storage(x, w.wdtype).reshape(rows, cols)
    return (draw(_S_WDOWN, w.D, w.r, w.D),
            draw(_S_WUP, w.r, w.H * w.dI, w.r),
            draw(_S_WW, w.D, w.H, w.D))


def all_layer_weights(w: ScoreWorkload, device="cpu"):
    """Stacked (W_down [L][D][r], W_up [L][r][H*dI], W_w [L][D][H])."""
    ws = [layer_weights(w, l, device) for l in range(w.L)]
    return tuple(torch.stack([x[i] for x in ws]) for i in range(3))


# ----------------------------------------------------------------------------- keys

def plant_fraction(w: ScoreWorkload, b: int) -> float:
    if w.plant_lo == w.plant_hi:
        return w.plant_lo
    key = rng.stream_key(w.seed, _S_FRAC)
    u = float(rng.uniform(key, torch.tensor([b], dtype=torch.int64))[0])
    return w.plant_lo + (w.plant_hi - w.plant_lo) * u


def planted(w: ScoreWorkload, b: int, start: int, n: int, device="cpu") -> torch.Tensor:
    """Bool [n]: which entries start..start+n-1 of sequence b are planted."""
    key = rng.stream_key(w.seed, _S_PLANT, b)
    return rng.uniform(key, rng.arange(n, start, device)) < plant_fraction(w, b)


def key_values(w: ScoreWorkload, b: int, l: int, direction, start: int, n: int,
               device="cpu") -> torch.Tensor:
    """fp64 key draws [n][dI] for entries start..start+n-1 of (b, l) before encoding."""
    key = rng.stream_key(w.seed, _S_KNOISE, b, l)
    idx = rng.arange(n * w.dI, start * w.dI, device)
    x = rng.normal(key, idx).reshape(n, w.dI)
    pl = planted(w, b, start, n, device)
    if bool(pl.any()):
        u = torch.as_tensor(direction, dtype=torch.float64, device=device).reshape(1, w.dI)
        x = torch.where(pl[:, None], 2.0 * u + math.sqrt(0.5) * x, x)
    return x


def encode_e4m3(x64: torch.Tensor):
    """Per-row scale and e4m3 codes: s = fp32(max|x|/448); codes = e4m3(x / s).

    Returns (codes uint8 [n][d], scale float32 [n]).  A row of zeros gets s = 1.
    """
    amax = x64.abs().amax(dim=1)
    s = (amax / E4M3_MAX).to(torch.float32)
    s = torch.where(s > 0, s, torch.ones_like(s))
    y = (x64 / s.to(torch.float64)[:, None]).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float32)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, s


def keys(w: ScoreWorkload, b: int, l: int, direction, start: int = 0, n: int | None = None,
         device="cpu"):
    """Encoded K_IComp rows of (b, l): (K [n][dI] in f32/bf16/uint8-e4m3, scale f32 [n] or None)."""
    if n is None:
        n = w.N - start
    x = key_values(w, b, l, direction, start, n, device)
    if w.kdtype == "e4m3":
        return encode_e4m3(x)
    return _to_storage(x, w.kdtype), None


def fine_query(w: ScoreWorkload, device="cpu"):
    """The backbone indexer's per-token query of each sequence for the fine selection
    inside the fetched subset: (q_f [B][H][dI] bf16 ~ N(0, 1), w_f [B][H] fp32 ~ N(0, 1)).
    The fine keys are a [B][N][dI] key array drawn like K_IComp (the benchmark reuses
    layer 0's keys for them)."""
    q = torch.empty(w.B, w.H, w.dI, dtype=torch.bfloat16, device=device)
    wv = torch.empty(w.B, w.H, dtype=torch.float32, device=device)
    for b in range(w.B):
        q[b] = _to_storage(rng.normal(rng.stream_key(w.seed, _S_FINE_Q, b), rng.arange(w.H * w.dI, device=device)),
                           "bf16").reshape(w.H, w.dI)
        wv[b] = rng.normal(rng.stream_key(w.seed, _S_FINE_W, b), rng.arange(w.H, device=device)).to(torch.float32)
    return q, wv


# ----------------------------------------------------------------------------- cold pool

def cold_rows(w: ScoreWorkload, b: int, start: int, n: int, device="cpu") -> torch.Tensor:
    """uint8 [n][row_bytes]: seeded contents of cold-pool rows start..start+n-1 of sequence b."""
    assert w.row_bytes % 4 == 0
    words = w.row_bytes // 4
    key = rng.stream_key(w.seed, _S_COLD, b)
    v = rng.u32(key, rng.arange(n * words, start * words, device))
    v = torch.where(v >= 2 ** 31, v - 2 ** 32, v).to(torch.int32)
    return v.view(torch.uint8).reshape(n, w.row_bytes)


# ----------------------------------------------------------------------------- vote logits

def vote_layers_boosted(v: VoteWorkload, p: int) -> list[int]:
    """The layers in which position p's boosted entries are boosted (sorted)."""
    nkey = rng.stream_key(v.seed, _S_VOTE_NLAYERS)
    m = v.min_layers + int(rng.u32(nkey, torch.tensor([p]))[0]) % (v.max_layers - v.min_layers + 1)
    lkey = rng.stream_key(v.seed, _S_VOTE_BOOST_LAYERS, p)
    order = torch.argsort(rng.u32(lkey, rng.arange(v.L)), stable=True)
    return sorted(int(x) for x in order[:m])


def vote_boost_set(v: VoteWorkload, p: int, device="cpu") -> torch.Tensor:
    """Sorted int64 indices of position p's boosted entries (round(boost_frac * N) of them)."""
    cnt = int(round(v.boost_frac * v.N))
    key = rng.stream_key(v.seed, _S_VOTE_BOOST_SET, p)
    hv = rng.u32(key, rng.arange(v.N, device=device))
    return torch.sort(torch.argsort(hv, stable=True)[:cnt]).values


def vote_logits(v: VoteWorkload, l: int, p: int, device="cpu", boost_set=None) -> torch.Tensor:
    """float32 [N] indexer logits of (layer l, position p)."""
    key = rng.stream_key(v.seed, _S_VOTE_X, l, p)
    x = rng.normal(key, rng.arange(v.N, device=device))
    if l in vote_layers_boosted(v, p):
        bs = vote_boost_set(v, p, device) if boost_set is None else boost_set
        x[bs] += v.boost
    return x.to(torch.float32)


def position_hidden(v: VoteWorkload, w: ScoreWorkload, device="cpu") -> torch.Tensor:
    """h [P][D] for the P query positions whose scores feed the label loss."""
    out = torch.empty(v.P, w.D, dtype=_torch_dtype(w.wdtype), device=device)
    for p in range(v.P):
        key = rng.stream_key(v.seed, _S_POS_H, p)
        out[p] = _to_storage(rng.normal(key, rng.arange(w.D, device=device)), w.wdtype)
    return out


# ----------------------------------------------------------------------------- stored params

def _f32_to_b64(t: torch.Tensor) -> str:
    return base64.b64encode(t.to(torch.float32).contiguous().numpy().tobytes()).decode()


def _b64_to_f32(s: str, shape) -> torch.Tensor:
    import numpy as np
    a = np.frombuffer(base64.b64decode(s), dtype="<f4").copy()
    return torch.from_numpy(a).reshape(shape)


def encode_params(bias: torch.Tensor, direction: torch.Tensor) -> dict:
    return {"bias": [float(x) for x in bias.to(torch.float32)],
            "direction_shape": list(direction.shape),
            "direction_f32_b64": _f32_to_b64(direction)}


def load_params(name: str, path: str = PARAMS_PATH):
    """(bias float32 [L], direction float32 [B][L][dI]) stored for workload `name`."""
    with open(path) as f:
        d = json.load(f)[name]
    bias = torch.tensor(d["bias"], dtype=torch.float32)
    direction = _b64_to_f32(d["direction_f32_b64"], d["direction_shape"])
    return bias, direction
