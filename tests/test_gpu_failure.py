"""Failure detection without a GPU fault: a bounded pipeline wait that runs out ends as a
status (the context stays usable), and an injected launch failure reaches the caller as
an error."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import lookahead_sparse_kv_score_b200 as lsa
from lookahead_sparse_kv_score_b200 import build
from oracle import lsa_oracle as O

import lsa_cases as C

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    build.build()
    lsa.lib()


def test_bounded_wait_gives_up_with_status_and_context_survives():
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    lsa.lsa_check_bounded_wait(20000, st)          # 20 ms on a barrier nothing arrives at
    b.record()
    torch.cuda.synchronize()
    assert int(st.item()) == lsa.LSA_ERR_TIMEOUT
    assert a.elapsed_time(b) >= 19.0
    # the context still works: a compaction right after gives the exact result
    g = np.random.default_rng(0)
    m = g.random((2, 3000)) < 0.2
    bits = torch.from_numpy(O.pack_bits(m).view(np.int32)).cuda()
    idx = torch.full((2, 3000), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(2, dtype=torch.int32, device="cuda")
    st.zero_()
    lsa.lsa_compact(2, 3000, bits, 3000, idx, cnt, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for r in range(2):
        e = O.compact(m[r])
        assert int(cnt[r]) == len(e) and np.array_equal(idx[r, : len(e)].cpu().numpy(), e)


def test_injected_launch_failure_reaches_the_caller():
    code = (
        "import torch, lookahead_sparse_kv_score_b200 as lsa\n"
        "m = torch.zeros(1, 4, dtype=torch.int32, device='cuda'); U = torch.zeros_like(m)\n"
        "try:\n"
        "    lsa.lsa_select_union(1, 4, m, U, None)\n"
        "    print('no error')\n"
        "except lsa.LsaError as e:\n"
        "    print('error', e.code, 'injected' in str(e))\n"
    )
    env = dict(os.environ, LSA_FAULT="launch", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert out.stdout.strip() == f"error {lsa.LSA_ERR_CUDA} True", out.stdout + out.stderr
