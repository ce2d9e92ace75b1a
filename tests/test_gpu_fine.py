"""Parity of lsa_fine_score (the native indexer's score of the fetched subset) and of the
fine top-k built on it with the fp64 oracle: tensor-core shapes (bf16 and e4m3 keys,
gathered rows), shapes that run on the CUDA cores, ragged and empty candidate lists,
lists longer than their capacity, and the 1M-context workload's own fetch lists in the
launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import build
from oracle import lsa_oracle as O
from oracle import step as OS
from synth import workloads as W

import lsa_cases as C

pytestmark = pytest.mark.gpu

# logit tolerance by key dtype (as for the lookahead score fed the oracle's query)
TZ = {"f32": 4e-5, "bf16": 8e-3, "e4m3": 4e-2}
KDT = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    lsa.lib()


def _keys(g, B, N, dI, kdt):
    """Key rows [B][N][dI] in storage form (and the e4m3 scale) from seeded normals."""
    x = torch.from_numpy(g.standard_normal((B * N, dI)))
    if kdt == "e4m3":
        codes, s = W.encode_e4m3(x)
        return codes.reshape(B, N, dI), s.reshape(B, N)
    return x.to(torch.float32).to(KDT[kdt]).reshape(B, N, dI), None


def _lists(g, B, N, cap, dens):
    idx = np.full((B, cap), -1, dtype=np.int32)
    cnt = np.zeros(B, dtype=np.int32)
    for b in range(B):
        e = np.flatnonzero(g.random(N) < dens[b]).astype(np.int32)
        cnt[b] = e.size                      # the true count; only cap indices are stored
        idx[b, : min(cap, e.size)] = e[:cap]
    return idx, cnt


def run_fine(q, w, K, ks, idx, cnt, cap, kdt, qdt=torch.bfloat16):
    B, N, dI = K.shape
    H = q.shape[1]
    dev = "cuda"
    score = torch.full((B, N), float("nan"), device=dev)
    kd = lsa.LSA_E4M3 if kdt == "e4m3" else lsa.dtype_code(KDT[kdt])
    ws = lsa.workspace(lsa.lsa_fine_score_workspace_bytes(B, H, dI, kd))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    lsa.lsa_fine_score(B, N, H, dI, lsa.dtype_code(qdt), q.to(qdt).to(dev).contiguous(), w.to(dev).contiguous(), kd,
                       K.to(dev).contiguous(), None if ks is None else ks.to(dev).contiguous(),
                       torch.from_numpy(idx).to(dev), cap, torch.from_numpy(cnt).to(dev), score, ws, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return score


def _oracle_scores(q, w, K, ks, kdt, b, entries):
    Kd = OS.decode_keys(C.raw(K[b]), None if ks is None else C.raw(ks[b]), kdt)
    return O.fine_index_scores(q[b].double().numpy(), w[b].double().numpy(), Kd, entries), Kd


def _check(q, w, K, ks, idx, cnt, cap, kdt, score, k=None):
    B, N = K.shape[0], K.shape[1]
    tz = TZ[kdt]
    sc = score.cpu().numpy()
    for b in range(B):
        n = min(int(cnt[b]), cap)
        ent = idx[b, :n].astype(np.int64)
        z, Kd = _oracle_scores(q, w, K, ks, kdt, b, ent)
        got = sc[b, ent].astype(np.float64)
        assert np.all(np.abs(got - z) <= tz), f"seq {b}: max error {np.max(np.abs(got - z)) if n else 0}"
        untouched = np.ones(N, dtype=bool)
        untouched[ent] = False
        assert np.isnan(sc[b, untouched]).all(), f"seq {b}: entries outside the list were written"
        if k is not None:
            want = O.fine_topk(q[b].double().numpy(), w[b].double().numpy(), Kd, ent, k)
            yield b, ent, z, want


def _topk(score, idx, cnt, cap, k):
    B, N = score.shape
    topk = torch.full((B, max(k, 1)), -9, dtype=torch.int32, device="cuda")
    tc = torch.zeros(B, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.lsa_topk_workspace_bytes(B, cap))
    cnt_d = torch.from_numpy(np.minimum(cnt, cap).astype(np.int32)).cuda()
    lsa.lsa_topk(B, 1, N, k, torch.from_numpy(idx).cuda(), cap, cnt_d, score, topk, tc, ws)
    torch.cuda.synchronize()
    return topk.cpu().numpy(), tc.cpu().numpy()


@pytest.mark.parametrize("kdt,H,dI", [("e4m3", 64, 128), ("bf16", 64, 128), ("e4m3", 32, 128), ("bf16", 128, 64)])
def test_fine_score_tensor_cores_and_fine_topk(kdt, H, dI):
    g = np.random.default_rng(H + dI)
    B, N, cap, k = 5, 9000, 9000, 300
    q = torch.from_numpy(g.standard_normal((B, H, dI))).to(torch.bfloat16)
    w = torch.from_numpy(g.standard_normal((B, H))).float()
    K, ks = _keys(g, B, N, dI, kdt)
    dens = [0.3, 0.0, 0.02, 1.0, 0.5]              # empty list, short list, every entry
    idx, cnt = _lists(g, B, N, cap, dens)
    score = run_fine(q, w, K, ks, idx, cnt, cap, kdt)
    checks = list(_check(q, w, K, ks, idx, cnt, cap, kdt, score, k=k))
    topk, tc = _topk(score, idx, cnt, cap, k)
    for b, ent, z, want in checks:
        n = ent.size
        assert tc[b] == min(k, n)
        got = topk[b, : tc[b]]
        if n == 0:
            continue
        kth = np.sort(z)[::-1][min(k, n) - 1]
        key = dict(zip(ent.tolist(), z.tolist()))
        diff = np.setxor1d(got, want)
        assert all(abs(key[int(e)] - kth) <= 2 * TZ[kdt] for e in diff), f"seq {b}: top-k differs outside the tie band"


@pytest.mark.parametrize("kdt,H,dI,qdt", [("f32", 8, 64, torch.float32), ("bf16", 48, 128, torch.bfloat16),
                                          ("e4m3", 64, 64, torch.bfloat16)])
def test_fine_score_cuda_core_shapes(kdt, H, dI, qdt):
    """Shapes the tensor-core path declines run on the CUDA cores with the same results."""
    g = np.random.default_rng(7 + H)
    B, N, cap = 3, 3000, 3000
    q = torch.from_numpy(g.standard_normal((B, H, dI))).to(qdt)
    w = torch.from_numpy(g.standard_normal((B, H))).float()
    K, ks = _keys(g, B, N, dI, kdt)
    idx, cnt = _lists(g, B, N, cap, [0.2, 0.05, 0.6])
    score = run_fine(q, w, K, ks, idx, cnt, cap, kdt, qdt=qdt)
    list(_check(q.float(), w, K, ks, idx, cnt, cap, kdt, score))


def test_fine_score_ragged_lists_and_capacity():
    """Counts that end mid-tile, a single candidate, and counts above cap (only the first
    cap candidates are scored)."""
    g = np.random.default_rng(3)
    B, N, H, dI, kdt = 6, 20000, 64, 128, "e4m3"
    cap = 700
    q = torch.from_numpy(g.standard_normal((B, H, dI))).to(torch.bfloat16)
    w = torch.from_numpy(g.standard_normal((B, H))).float()
    K, ks = _keys(g, B, N, dI, kdt)
    idx = np.full((B, cap), -1, dtype=np.int32)
    cnt = np.array([1, 129, 127, 700, 5000, 0], dtype=np.int32)
    for b in range(B):
        e = np.sort(g.choice(N, size=int(cnt[b]), replace=False)).astype(np.int32)
        idx[b, : min(cap, e.size)] = e[:cap]
    score = run_fine(q, w, K, ks, idx, cnt, cap, kdt)
    list(_check(q, w, K, ks, idx, cnt, cap, kdt, score))


def test_fine_score_full_size_1m_fetch_lists():
    """The 1M-context workload's fetch lists (the union of the three layers, ~70K entries
    per sequence, B = 32) scored by the native indexer with layer 0's keys standing in for
    its own, as the benchmark runs it: every scored entry and the fine top-2048 of
    sequences 0, 13 and 31, and 512 sampled scores of every other sequence, against the
    oracle."""
    import bench
    w = W.WORKLOADS["lsa_step_1m_b32_fp8"]
    dev = torch.device("cuda")
    inp = bench.device_inputs(w, dev)
    trig = bench.Trigger(lsa, w, inp, None, dev)
    trig.select_only()
    torch.cuda.synchronize()
    qf, wf = W.fine_query(w)
    K0, ks0 = inp["K"][0], inp["kscale"][0]
    cnt = trig.cnt_U.cpu().numpy()
    idx = trig.idx_U.cpu().numpy()
    score = run_fine(qf, wf, K0, ks0, idx, cnt, w.N, "e4m3")
    topk, tc = _topk(score, idx, cnt, w.N, w.k)
    sc = score.cpu().numpy()
    K0h, ks0h = C.raw(K0), C.raw(ks0)
    del trig, inp
    for b in range(w.B):
        n = int(cnt[b])
        ent = idx[b, :n].astype(np.int64)
        full = b in (0, 13, 31)
        rows = ent if full else np.sort(ent[np.random.default_rng(b).choice(n, size=min(n, 512), replace=False)])
        Kd = OS.decode_keys(K0h[b][rows], ks0h[b][rows], "e4m3")
        z = O.fine_index_scores(qf[b].double().numpy(), wf[b].double().numpy(), Kd, np.arange(rows.size))
        assert np.all(np.abs(sc[b, rows] - z) <= TZ["e4m3"]), b
        if full:
            key = np.full(w.N, -np.inf)
            key[ent] = z
            want = O.topk_in_fetched(ent, key, w.k)
            kth = np.sort(z)[::-1][min(w.k, n) - 1]
            got = topk[b, : tc[b]]
            assert tc[b] == min(w.k, n)
            diff = np.setxor1d(got, want)
            assert np.all(np.abs(key[diff] - kth) <= 2 * TZ["e4m3"]), b
