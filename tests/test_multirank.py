"""The N>1 path on CPU: two gloo ranks exercise the bench's replica logic
(weak scaling, no collective on the data path; the only collectives are the
timing reductions and barriers).  No GPU."""
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
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ws, r, lr = bench.dist_env()
    assert (ws, r, lr) == (world, rank, rank)
    # per-rank elapsed times differ; the reported time is the max over ranks
    t = bench.max_over_ranks(10.0 + rank, ws)
    tot = bench.sum_over_ranks(2.0 ** rank, ws)
    bench.barrier(ws)
    # every rank builds its own replica of the workload from its own seed:
    # the problems are independent (no data exchange)
    import workloads as W
    p = W.paged_uniform(num_seqs=3, H=2, d=8, block_size=16, pool=64, len_lo=1, len_hi=200, seed=rank)
    out[rank] = (t, tot, int(p.seq_lens.sum()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timing_and_run_independent_replicas():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 11.0
    assert out[0][1] == out[1][1] == 3.0
    assert out[0][2] != out[1][2]  # different seeds -> different replicas


def test_reference_arm_only_rank0(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert capsys.readouterr().out == ""
