"""Multi-rank bookkeeping of bench.py on CPU (gloo, world size 2).

The Sign-Muon path runs as independent replicas on N GPUs (the M workers are
buffers on one GPU, so there is no exchange step); what N > 1 adds is the
timing: every rank times its own steps and the job is timed by the slowest
rank.  This checks that reduction and the aggregate on two gloo ranks."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = [120.0, 150.0][rank]
    mx = bench.max_over_ranks_value(local_ms, world, "cpu")
    value = bench.job_throughput(1000, 10, world, mx)
    out[rank] = (mx, value)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 150.0
    assert res[0][1] == pytest.approx(1000 * 10 * 2 / 0.150)
    assert res[0] == res[1]


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks_value(3.5, 1, "cpu") == 3.5
    assert bench.job_throughput(10, 4, 1, 2000.0) == pytest.approx(20.0)
