"""The parity bounds of the projection, checked on the CPU against simulated fp32
arithmetic: a projection that sums in fp32 in slices (the CUDA-core layout: 256-element
slices added in order; a tensor-core-like layout: 512-element slices in an arbitrary
order) and rounds c and q to bf16 must stay within the per-element bound the GPU parity
tests allow (tests/lsa_cases.py, q_allowed and w_allowed).

That bound is rigorous for any summation order up to its depth, and therefore loose: a
worst-case fp32 error of 1100 additions, which marks nearly every element of c as one
that may round the other way, comes to about 16 bf16 ulps of q at the median.  The
simulated devices themselves land within one ulp of the oracle everywhere and on it
almost everywhere, which is what a tighter statistical check of the device's q could ask.
"""
import numpy as np
import pytest
import torch

from oracle import step as OS
from synth import workloads as W

import lsa_cases as C


def _bf16(x32: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 (ties to even), returned as float32 values."""
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _sliced_sum(terms: np.ndarray, slice_len: int, rng=None) -> np.ndarray:
    """Sum terms [K][M] over K in fp32: sequential sums over slices of slice_len (in a
    random order within each slice when rng is given), then the slice sums in order."""
    K, M = terms.shape
    ns = -(-K // slice_len)
    pad = np.zeros((ns * slice_len, M), dtype=np.float32)
    pad[:K] = terms
    sl = pad.reshape(ns, slice_len, M)
    if rng is not None:
        sl = np.take_along_axis(sl, np.argsort(rng.random(sl.shape), axis=1), axis=1)
    part = np.cumsum(sl, axis=1, dtype=np.float32)[:, -1, :]
    return np.cumsum(part, axis=0, dtype=np.float32)[-1]


@pytest.fixture(scope="module")
def case():
    w = W.scaled(W.WORKLOADS["lsa_step_128k_b1_bf16"], L=1, N=64)
    inp = C.make_inputs(w, device="cpu")
    return w, C.OracleCache(inp)


@pytest.mark.parametrize("layout", ["cuda_cores", "tensor_cores"])
def test_simulated_fp32_projection_within_the_parity_bound(case, layout):
    w, orc = case
    rng = np.random.default_rng(0) if layout == "tensor_cores" else None
    slice_len = 256 if layout == "cuda_cores" else 512
    h = OS.decode(orc._h[0, 0], w.wdtype).astype(np.float32)
    Wd = OS.decode(orc._Wd[0], w.wdtype).astype(np.float32)
    Wu = OS.decode(orc._Wu[0], w.wdtype).astype(np.float32)
    Ww = OS.decode(orc._Ww[0], w.wdtype).astype(np.float32)
    # products of two bf16 values are exact in fp32; only the sums round
    c = _bf16(_sliced_sum(h[:, None] * Wd, slice_len, rng))
    q = _bf16(_sliced_sum(c[:, None] * Wu, slice_len, rng)).reshape(w.H, w.dI)
    wv = _sliced_sum(h[:, None] * Ww, slice_len, rng)
    q_o, w_o = orc.qw(0, 0)
    allowed = orc.q_allowed(0, 0)
    assert np.all(np.abs(q.astype(np.float64) - q_o) <= allowed)
    assert np.all(np.abs(wv.astype(np.float64) - w_o) <= orc.w_allowed(0, 0))
    ulp = C.bf16_ulp(q_o)
    # the rigorous bound's looseness, recorded: ~16 ulps of q at the median
    assert 4.0 < np.median(allowed / ulp) < 32.0, np.median(allowed / ulp)
    # what an fp32 device actually achieves: within one ulp everywhere, equal almost everywhere
    d = np.abs(q.astype(np.float64) - q_o) / ulp
    assert d.max() <= 1.0 and np.mean(d > 0) < 0.01, (d.max(), np.mean(d > 0))
