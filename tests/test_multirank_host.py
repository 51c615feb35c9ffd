"""World-size-2 checks of bench.py's multi-rank host logic on CPU (gloo).

By default the ranks split one layer's kv heads and all-gather the outputs
(strong scaling); with --shard layers they run independent layers (weak
scaling, no exchange on the data path).  The collectives are the barrier, the
max over ranks of the timed region and the output gather, which these tests
exercise without a GPU.
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


def _fake_prefill(q, k, v, block_size, params):
    """Stand-in for the library call (no GPU here): a per-head function of the
    head's own q and its kv head's k and v, so that a wrong slice shows."""
    g = q.shape[1] // k.shape[1]
    kk = k.repeat_interleave(g, dim=1)
    vv = v.repeat_interleave(g, dim=1)
    return 2.0 * q + 3.0 * kk - vv, None, None


def _shard_worker(rank, ws, port, out):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from dynamic_block_sparse_fp_b200 import ops, sharded
    dist.init_process_group("gloo", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ops.prefill_attn = _fake_prefill  # this process only
        g = torch.Generator().manual_seed(3)
        q = torch.randn(2, 8, 16, 4, generator=g)   # Bt 2, Hq 8
        k = torch.randn(2, 4, 16, 4, generator=g)   # Hkv 4: 2 kv heads per rank
        v = torch.randn(2, 4, 16, 4, generator=g)
        full = sharded.sharded_prefill_attn(q, k, v, 8, None)
        local = sharded.sharded_prefill_attn(q, k, v, 8, None, gather=False)
        want = _fake_prefill(q, k, v, 8, None)[0]
        kv0, nk = sharded.head_shard(4, ws, rank)
        out[rank] = (bool(torch.equal(full, want)),
                     bool(torch.equal(local, want[:, kv0 * 2:(kv0 + nk) * 2])))
    finally:
        dist.destroy_process_group()


def test_two_ranks_head_sharded_layer_gathers_every_head():
    ws = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_shard_worker, args=(ws, _free_port(), out), nprocs=ws, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0] == res[1] == (True, True)


def test_head_shard_rule():
    from dynamic_block_sparse_fp_b200 import sharded
    assert [sharded.head_shard(8, 4, r) for r in range(4)] == [(0, 2), (2, 2), (4, 2), (6, 2)]
    assert sharded.head_shard(8, 1, 0) == (0, 8)
    with pytest.raises(ValueError):
        sharded.head_shard(8, 3, 0)
    with pytest.raises(ValueError):
        sharded.head_shard(8, 2, 2)


def test_bench_splits_heads_by_default():
    import bench
    assert bench.parser().parse_args([]).shard == "heads"
    assert bench.parser().parse_args(["--shard", "layers"]).shard == "layers"


@pytest.mark.parametrize("bt", [1, 3])
def test_gathered_heads_layout(bt):
    """all_gather_into_tensor leaves [world, Bt, h, N, d]; the gathered layer is
    [Bt, world*h, N, d] in rank order (a view without a copy when Bt = 1)."""
    from dynamic_block_sparse_fp_b200 import sharded
    world, h = 4, 2
    parts = [torch.randn(bt, h, 5, 3) for _ in range(world)]
    buf = torch.stack(parts)
    got = sharded.heads_of_gathered(buf)
    assert torch.equal(got, torch.cat(parts, dim=1))
    if bt == 1:
        assert got.data_ptr() == buf.data_ptr()
