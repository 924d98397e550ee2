"""World-size-2 gloo check of bench.py's multi-process plumbing (replicas,
barrier, max-over-ranks timing).  CPU only: no GPU and no collective on the
data path."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(dist)
    local_ms = 10.0 + 5.0 * rank                      # the slower rank decides the job time
    out[rank] = bench.max_over_ranks(local_ms, dist, "cpu")
    bench.barrier(dist)
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == pytest.approx(15.0) and out[1] == pytest.approx(15.0)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
