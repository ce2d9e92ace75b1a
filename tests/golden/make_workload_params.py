"""Writes tests/golden/workload_params.json: per workload, the planted-key direction of
every (sequence, layer) and the per-layer bias.  Calls only the generator (``synth``)
and the oracle (``oracle``); nothing from the CUDA path.

  direction[b][l] = unit(mean over heads of the oracle's query q_h)   (fp32)
  bias[l]         = the oracle's bias that puts 10% of a calibration sample of
                    pre-bias logits at or above 0 (fp32); the sample is the first
                    min(N, 8192) entries of every sequence of that layer.

Run from the repository root:  python tests/golden/make_workload_params.py
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import step as OS            # noqa: E402
from oracle import lsa_oracle as O       # noqa: E402
from synth import workloads as W         # noqa: E402

CALIB_ENTRIES = 8192
TARGET_FRACTION = 0.10


def raw(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def workload_params(w: W.ScoreWorkload):
    h = W.hidden_states(w)
    Wd, Wu, Ww = W.all_layer_weights(w)
    direction = np.zeros((w.B, w.L, w.dI))
    qs = {}
    for b in range(w.B):
        for l in range(w.L):
            q, wv = OS.project(raw(h[b, l]), raw(Wd[l]), raw(Wu[l]), raw(Ww[l]), w.H, w.dI, w.wdtype)
            m = q.mean(axis=0)
            direction[b, l] = m / np.linalg.norm(m)
            qs[b, l] = (q, wv)
    direction = direction.astype(np.float32)
    n = min(w.N, CALIB_ENTRIES)
    bias = np.zeros(w.L)
    for l in range(w.L):
        zs = []
        for b in range(w.B):
            K, s = W.keys(w, b, l, torch.from_numpy(direction[b, l]).double(), 0, n)
            z, _, _ = OS.score_layer(qs[b, l][0], qs[b, l][1], 0.0, raw(K),
                                     None if s is None else s.numpy(), w.kdtype)
            zs.append(z)
        bias[l] = O.bias_for_fraction(np.concatenate(zs), TARGET_FRACTION)
    return torch.from_numpy(bias.astype(np.float32)), torch.from_numpy(direction)


def main(names=None):
    path = W.PARAMS_PATH
    out = {}
    if os.path.exists(path):
        with open(path) as f:
            out = json.load(f)
    for name, w in W.WORKLOADS.items():
        if names and name not in names:
            continue
        bias, direction = workload_params(w)
        out[name] = W.encode_params(bias, direction)
        print(name, "bias", [round(float(x), 4) for x in bias], flush=True)
    with open(path, "w") as f:
        json.dump(out, f, indent=1, sort_keys=True)
        f.write("\n")


if __name__ == "__main__":
    main(sys.argv[1:] or None)
