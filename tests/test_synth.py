"""The seeded generators: determinism, slice independence, distributions, and that the
stored workload parameters are what the oracle-only script writes."""
import os
import sys

import numpy as np
import pytest
import torch

from synth import rng
from synth import workloads as W

HERE = os.path.dirname(__file__)


def test_hash_is_deterministic_and_slices_agree():
    key = rng.stream_key(5, 1, 2)
    a = rng.u32(key, rng.arange(1000))
    b = rng.u32(key, rng.arange(500, 500))
    assert torch.equal(a[500:], b)
    assert int(a.min()) >= 0 and int(a.max()) < 2 ** 32
    assert not torch.equal(a, rng.u32(rng.stream_key(5, 1, 3), rng.arange(1000)))


def test_fmix32_matches_integer_reference():
    xs = [0, 1, 2, 0xDEADBEEF, 0xFFFFFFFF, 123456789]
    t = rng.fmix32(torch.tensor(xs, dtype=torch.int64))
    assert [int(v) for v in t] == [rng._fmix32_int(x) for x in xs]


def test_normals_moments():
    x = rng.normal(rng.stream_key(9), rng.arange(1 << 20))
    assert abs(float(x.mean())) < 0.005
    assert abs(float(x.std()) - 1.0) < 0.005
    assert float(x.abs().max()) < 7.0


def test_keys_planted_fraction_and_encoding():
    w = W.scaled(W.WORKLOADS["lsa_step_1m_b32_fp8"], N=20000)
    u = torch.zeros(w.dI, dtype=torch.float64)
    u[0] = 1.0
    pl = W.planted(w, 3, 0, w.N)
    f = W.plant_fraction(w, 3)
    assert 0.02 <= f <= 0.15
    assert abs(float(pl.double().mean()) - f) < 0.01
    codes, s = W.keys(w, 3, 0, u, 0, w.N)
    assert codes.dtype == torch.uint8 and s.dtype == torch.float32
    x = codes.view(torch.float8_e4m3fn).double() * s.double()[:, None]
    ref = W.key_values(w, 3, 0, u, 0, w.N)
    # per-entry scale maps the row max to 448; e4m3 keeps 4 significant bits
    assert float((x - ref).abs().max() / ref.abs().max()) < 2 ** -4
    assert float(codes.view(torch.float8_e4m3fn).double().abs().amax(dim=1).min()) == 448.0
    # planted entries lean on the direction: mean of component 0 is ~2 there
    assert float(ref[pl, 0].mean()) > 1.5 and abs(float(ref[~pl, 0].mean())) < 0.1


def test_cold_rows_deterministic():
    w = W.WORKLOADS["lsa_step_128k_b1_bf16"]
    a = W.cold_rows(w, 0, 10, 5)
    b = W.cold_rows(w, 0, 12, 2)
    assert a.shape == (5, w.row_bytes) and torch.equal(a[2:4], b)


def test_vote_generator_shape():
    v = W.VOTE_WORKLOADS["vote_labels_l24_p64_n131072"]
    for p in range(5):
        ls = W.vote_layers_boosted(v, p)
        assert 3 <= len(ls) <= 8 and all(0 <= l < 24 for l in ls)
    bs = W.vote_boost_set(v, 0)
    assert len(bs) == 1311 and len(set(bs.tolist())) == 1311


def test_stored_params_reproduce_from_oracle_script():
    sys.path.insert(0, os.path.join(HERE, "golden"))
    import make_workload_params as M
    for name in ("lsa_step_16k_tiny_fp32", "lsa_step_128k_b1_bf16"):
        bias, direction = M.workload_params(W.WORKLOADS[name])
        sb, sd = W.load_params(name)
        assert torch.equal(bias, sb) and torch.equal(direction, sd)
