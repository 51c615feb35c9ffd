"""World-size-2 checks of bench.py's multi-rank host logic on CPU (gloo).

Ranks run independent layers (weak scaling, no exchange on the data path);
the only collectives are the barrier and the max over ranks of the timed
region, which these tests exercise without a GPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, ws, port, out):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    import bench
    from dynamic_block_sparse_fp_b200 import synth
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(10.0 * (rank + 1), ws, "cpu")
        bench.barrier(ws)
        w = synth.WORKLOADS["tiny_n1024"]
        wr = bench.rank_workload(w, rank)
        q = synth.make_inputs(wr)["q"]
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(ws)]
        dist.all_gather(sums, q.double().sum().reshape(1))
        out[rank] = (t, wr.seed, [float(x) for x in sums])
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_timing_and_independent_layers():
    ws = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(ws, _free_port(), out), nprocs=ws, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 20.0  # the slowest rank's time on every rank
    assert res[0][1] != res[1][1]          # each rank its own seed
    assert res[0][2][0] != res[0][2][1]    # ... and its own data


def test_job_value_is_whole_job_tokens_per_second():
    import bench
    assert bench.job_value(131072, 1, 100.0) == pytest.approx(1310720.0)
    assert bench.job_value(131072, 8, 100.0) == pytest.approx(8 * 1310720.0)
    w = __import__("dynamic_block_sparse_fp_b200.synth", fromlist=["x"]).WORKLOADS["tiny_n1024"]
    assert bench.rank_workload(w, 0) is w
