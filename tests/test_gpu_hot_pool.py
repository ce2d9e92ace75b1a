"""Parity of lsa_hot_pool_update (residency across triggers) with the oracle's HotPool:
slot maps, stamps, resident bits and moved counts bit-exact, hot rows byte-exact."""
import numpy as np
import pytest
import torch

import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import build
from oracle import lsa_oracle as O

import lsa_cases as C

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    lsa.lib()


class Pool:
    def __init__(self, B, N, slots, R, seed):
        g = np.random.default_rng(seed)
        self.B, self.N, self.slots, self.R = B, N, slots, R
        self.cold = torch.from_numpy(g.integers(0, 256, size=(B, N, R), dtype=np.uint8)).pin_memory()
        self.hot = torch.zeros(B, slots, R, dtype=torch.uint8, device="cuda")
        self.state = lsa.workspace(lsa.lsa_hot_pool_state_bytes(B, N, slots))
        self.ws = lsa.workspace(lsa.lsa_hot_pool_workspace_bytes(B, N, slots))
        self.off = lsa.lsa_hot_pool_layout(B, N, slots)
        self.moved = torch.full((B,), -1, dtype=torch.int32, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        lsa.lsa_hot_pool_reset(B, N, slots, self.state)
        self.oracle = [O.HotPool(N, slots) for _ in range(B)]
        self.ohot = np.zeros((B, slots, R), dtype=np.uint8)

    def update(self, sets, t):
        marks = np.zeros((self.B, self.N), dtype=bool)
        for b, U in enumerate(sets):
            marks[b, list(U)] = True
        U = torch.from_numpy(O.pack_bits(marks).view(np.int32)).cuda()
        self.status.zero_()
        lsa.lsa_hot_pool_update(self.B, self.N, self.slots, self.R, t, U, self.cold, self.hot, self.state,
                                self.moved, self.status, self.ws)
        torch.cuda.synchronize()
        exp = [self.oracle[b].update(sets[b], t, self.cold[b].numpy(), self.ohot[b]) for b in range(self.B)]
        return exp

    def array(self, i, dtype, shape):
        n = int(np.prod(shape)) * 4
        return self.state[self.off[i]: self.off[i] + n].view(dtype).reshape(shape).cpu().numpy()

    def check(self, exp):
        B, N, slots = self.B, self.N, self.slots
        slot_of = self.array(0, torch.int32, (B, N))
        entry_of = self.array(1, torch.int32, (B, slots))
        stamp = self.array(2, torch.int32, (B, slots)).view(np.uint32)
        resident = C.unpack(torch.from_numpy(self.array(3, torch.int32, (B, (N + 31) // 32))), N)
        moved = self.moved.cpu().numpy()
        hot = self.hot.cpu().numpy()
        for b in range(B):
            o = self.oracle[b]
            assert np.array_equal(slot_of[b], o.slot_of), b
            assert np.array_equal(entry_of[b], o.entry_of), b
            assert np.array_equal(stamp[b], np.array(o.stamp, dtype=np.uint32)), b
            assert np.array_equal(resident[b], np.array(o.slot_of) >= 0), b
            assert moved[b] == (0 if exp[b] is None else len(exp[b])), b
            used = np.array(o.entry_of) >= 0
            assert np.array_equal(hot[b][used], self.ohot[b][used]), b
        return int(self.status.item())


def drift(g, N, prev, size, keep):
    kept = [e for e in prev if g.random() < keep]
    rest = np.setdiff1d(np.arange(N), np.array(kept, dtype=np.int64))
    new = g.choice(rest, size=max(0, size - len(kept)), replace=False)
    return set(kept) | set(int(e) for e in new)


def test_hot_pool_drifting_fetch_sets():
    """Three sequences over twelve triggers; fetch sets drift (70-90% kept), one trigger
    of sequence 1 exceeds the pool and must move nothing."""
    g = np.random.default_rng(0)
    B, N, slots, R = 3, 5000, 700, 64
    p = Pool(B, N, slots, R, 1)
    sets = [set() for _ in range(B)]
    for t in range(1, 13):
        for b in range(B):
            size = int(g.integers(200, 650))
            if b == 1 and t == 7:
                size = slots + 50
            sets[b] = drift(g, N, sets[b], size, keep=0.7 + 0.1 * b)
        exp = p.update(sets, t)
        st = p.check(exp)
        assert st == (lsa.LSA_ERR_CAPACITY if t == 7 else 0), t


def test_hot_pool_single_entry_triggers_lru():
    """One entry per trigger: the pool behaves as an LRU cache (checked by the oracle)."""
    g = np.random.default_rng(2)
    B, N, slots, R = 2, 64, 5, 16
    p = Pool(B, N, slots, R, 3)
    for t in range(1, 60):
        exp = p.update([{int(g.integers(0, N))} for _ in range(B)], t)
        assert p.check(exp) == 0


def test_hot_pool_full_size_sequences():
    """32 sequences of 2^18 entries and 100,000 slots (a cluster of CTAs per sequence in
    the slot selection), three triggers with ~70,000-entry fetch sets."""
    g = np.random.default_rng(4)
    B, N, slots, R = 32, 262144, 100000, 16
    p = Pool(B, N, slots, R, 5)
    sets = [set() for _ in range(B)]
    for t in range(1, 4):
        sets = [drift(g, N, sets[b], int(g.integers(60000, 80000)), keep=0.8) for b in range(B)]
        exp = p.update(sets, t)
        assert p.check(exp) == 0


def test_hot_pool_more_sequences_than_one_launch():
    """4,500 sequences: the move step runs in blocks of 4,096 sequences; one sequence of
    the second block overflows the pool on trigger 2 and must move nothing."""
    g = np.random.default_rng(6)
    B, N, slots, R = 4500, 64, 16, 16
    p = Pool(B, N, slots, R, 7)
    sets = [set() for _ in range(B)]
    for t in range(1, 4):
        sets = [drift(g, N, sets[b], int(g.integers(0, slots + 1)), keep=0.6) for b in range(B)]
        if t == 2:
            sets[4400] = set(range(slots + 3))
        exp = p.update(sets, t)
        assert p.check(exp) == (lsa.LSA_ERR_CAPACITY if t == 2 else 0), t
