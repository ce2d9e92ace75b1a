"""Tensor-core scoring (tcgen05 + TMA) against the oracle: fp8 keys with the split query,
shapes that fall back to the CUDA-core path, and the full-size workloads in the launch
configuration the benchmark times (sampled entries against the oracle, invariants on
every entry)."""
import numpy as np
import pytest
import torch

import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import build
from synth import workloads as W

import lsa_cases as C
from test_gpu_score import check_layer_outputs, oracle_query_tensors, run_score

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    lsa.lib()


@pytest.mark.parametrize("N", [5000, 128, 77])
def test_fp8_keys_with_oracle_query(N):
    w = W.scaled(W.WORKLOADS["lsa_step_1m_b32_fp8"], B=3, N=N)
    inp = C.make_inputs(w)
    orc = C.OracleCache(inp)
    q_in, w_in = oracle_query_tensors(inp, orc)
    out = run_score(inp, q_in=q_in, w_in=w_in, want_q=False)
    for l in range(w.L):
        for b in range(w.B):
            check_layer_outputs(out, inp, orc, l, b)


def test_fp8_end_to_end_with_query_bound():
    w = W.scaled(W.WORKLOADS["lsa_step_1m_b32_fp8"], B=2, N=3000)
    inp = C.make_inputs(w)
    orc = C.OracleCache(inp)
    out = run_score(inp)
    for l in range(w.L):
        for b in range(w.B):
            check_layer_outputs(out, inp, orc, l, b, z_extra=orc.z_bound_from_q(l, b))


@pytest.mark.parametrize("H,dI,kdt", [(48, 128, "bf16"), (64, 64, "e4m3"), (32, 64, "bf16"), (64, 256, "bf16")])
def test_other_shapes(H, dI, kdt):
    """Shapes the tensor-core path declines (H=48, e4m3 with dI=64) run on the CUDA
    cores; (32, 64) and (64, 256) exercise other tensor-core tile shapes."""
    base = W.WORKLOADS["lsa_step_512k_b8_bf16"]
    w = W.scaled(base, name="lsa_step_512k_b8_bf16", B=2, N=2000, H=H, dI=dI, kdtype=kdt, r=128, D=256)
    bias = torch.tensor([-20.0, -20.0, -20.0])
    direction = torch.nn.functional.normalize(torch.ones(w.B, w.L, dI), dim=-1)
    inp = C.make_inputs_with(w, bias, direction)
    orc = C.OracleCache(inp)
    q_in, w_in = oracle_query_tensors(inp, orc)
    out = run_score(inp, q_in=q_in, w_in=w_in, want_q=False)
    for l in range(w.L):
        for b in range(w.B):
            check_layer_outputs(out, inp, orc, l, b)


def test_all_layers_in_one_launch_equals_per_layer():
    w = W.scaled(W.WORKLOADS["lsa_step_512k_b8_bf16"], B=3, N=10000)
    inp = C.make_inputs(w)
    a = run_score(inp, want_q=False)
    per = [run_score(inp, layer=l, want_q=False) for l in range(w.L)]
    for l in range(w.L):
        assert torch.equal(a["mask"][l], per[l]["mask"][l])
        assert torch.equal(a["logit"][l], per[l]["logit"][l])


def _full_size_check(name, samples_per_unit=192, seqs=None):
    """Full-size workload, all layers in one launch as the benchmark runs it.
    (1) with the oracle's query: sampled logits within the tolerance, sampled mask bits
        exact outside the band; (2) with the projection inside the call: every query
        element within the rigorous fp32 bound of the oracle's (q_allowed) and the mask
        consistent with the logits on every entry."""
    w = W.WORKLOADS[name]
    inp = C.make_inputs(w)
    orc = C.OracleCache(inp)
    g = np.random.default_rng(0)
    units = [(l, b) for l in range(w.L) for b in (range(w.B) if seqs is None else seqs)]
    q_in, w_in = oracle_query_tensors(inp, orc)
    out = run_score(inp, q_in=q_in, w_in=w_in, want_q=False)
    for l, b in units:
        ent = np.unique(np.concatenate([np.arange(128), np.arange(w.N - 128, w.N),
                                        g.choice(w.N, samples_per_unit, replace=False)]))
        et = torch.from_numpy(ent).cuda()
        z = orc.z(l, b, et)
        tz = C.tol_z(w.kdtype)
        zs = out["logit"][l, b][et].double().cpu().numpy()
        assert np.all(np.abs(zs - z) <= tz), f"({l},{b}) max logit error {np.max(np.abs(zs - z))}"
        bits = C.unpack(out["mask"][l, b], w.N)
        assert not ((bits[ent] != (z >= 0)) & (np.abs(z) > tz)).any()
    del out
    out = run_score(inp, want_q=True)
    marked = {l: [] for l in range(w.L)}
    for l, b in units:
        q, _ = orc.qw(l, b)
        assert C.q_within(out["q"][l, b].double().cpu().numpy(), q, orc.q_allowed(l, b)).all()
        bits = C.unpack(out["mask"][l, b], w.N)
        assert np.array_equal(bits, (out["logit"][l, b] >= 0).cpu().numpy())
        marked[l].append(bits.mean())
    # the bias is calibrated on pooled sequences (10% of a sample); single sequences vary
    for l in range(w.L):
        assert 0.02 < float(np.mean(marked[l])) < 0.3, marked[l]
    return out


def test_full_size_512k_b8_bf16_sampled():
    _full_size_check("lsa_step_512k_b8_bf16")


def test_full_size_1m_b32_fp8_sampled():
    _full_size_check("lsa_step_1m_b32_fp8", samples_per_unit=96, seqs=[0, 7, 31])
