"""Multi-GPU host logic of bench.py on CPU: two gloo ranks.

With N GPUs every rank runs an independent replica (decode shards by
sequence; no collective on the data path).  The only exchanges are the
timing reductions: the job's device time is the slowest rank's, and the
job's throughput counts the tokens of every rank.  The reference leg runs
on rank 0 alone."""
import datetime
import os
import socket
import types

import pytest
import torch.multiprocessing as mp

import bench
from compressed_sparse_attention_topk_b200 import workloads as wl


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    w, r, local = bench.dist_env()
    # per-rank device times (ms) of the timed region and of the end-to-end pass
    times = bench.max_over_ranks(dist, [10.0 + rank, 5.0 - rank], torch.device("cpu"))
    value = bench.job_tokens_per_s(w, 50, 4, 1, 2, times[0])
    dist.barrier()
    dist.destroy_process_group()
    queue.put((rank, w, r, local, times, value))


def test_two_ranks_take_the_slowest_rank_time_and_count_every_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(60)
    assert all(p.exitcode == 0 for p in procs)
    for rank, w, r, local, times, value in results:
        assert (w, r, local) == (2, rank, rank)
        assert times == [11.0, 5.0]                      # element-wise max over ranks
        assert value == pytest.approx(2 * 50 * 4 * 1 * 2 / 11e-3)


def test_single_process_needs_no_collective():
    assert bench.max_over_ranks(None, [3.5, 7], None) == [3.5, 7.0]
    assert bench.job_tokens_per_s(1, 10, 4, 1, 2, 1.0) == pytest.approx(80_000.0)


def test_reference_leg_runs_on_rank_0_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = types.SimpleNamespace(steps=1, warmup=0, gpus=2)
    assert bench.run_reference(args, wl.TINY) == 0
    assert capsys.readouterr().out == ""
