"""The multi-rank host logic of bench.py on CPU: two gloo ranks, whole-job aggregation
(units summed, time = max over ranks) and the reference arm running on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    dev = torch.device("cpu")
    units, ms, value = bench.whole_job(1000 * (rank + 1), 10.0 * (rank + 1), dist, dev)
    bench.barrier(dist, dev)
    out[rank] = (units, ms, value)
    # the reference arm runs on rank 0 only; other ranks return at once without work
    if rank == 1:
        out[2] = bench.reference_arm(bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"]))
    dist.destroy_process_group()


def test_two_rank_aggregation_and_reference_rank_gate():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    for r in (0, 1):
        units, ms, value = out[r]
        assert units == 3000 and ms == 20.0                 # sum of units, max of times
        assert value == pytest.approx(3000 / 0.020)
    assert out[2] == 0
