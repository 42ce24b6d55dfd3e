"""World-size-2 gloo checks of the multi-GPU host logic (CPU only).

Attention heads are independent, so the multi-GPU path has no data-path
collective: every rank runs its own per-GPU workload (weak scaling) and the
benchmark only needs a barrier and the max of the per-rank times.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier(world)
        got = bench._max_over_ranks(10.0 + rank, world)
        # each rank draws its own inputs (seed + rank): different data, same shapes
        from exact_io_aware_84_b200.inputs import make_inputs, workload
        w = workload("tiny_fwd")
        x = make_inputs(w.with_(seed=w.seed + rank), with_grad=False)
        gathered = [torch.zeros_like(x["q"].float()) for _ in range(world)]
        dist.all_gather(gathered, x["q"].float())
        out[rank] = (got, bool(torch.equal(gathered[0], gathered[1])), tuple(x["q"].shape))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_independent_shards():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        got, same, shape = out[r]
        assert got == 11.0            # max over ranks, seen by every rank
        assert not same               # ranks hold different data
        assert shape == (1, 1, 256, 64)


def test_reference_arm_non_zero_rank_exits_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        workload = "tiny_fwd"
        steps = 1
        warmup = 0
    assert bench.run_reference(A) == 0
    assert capsys.readouterr().out == ""
