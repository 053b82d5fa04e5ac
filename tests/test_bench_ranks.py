"""The bench's multi-process plumbing on CPU: two gloo ranks (replicas; no data-path collective).

Every rank must end with the slowest rank's time (max over ranks), and the rank / world / local
rank come from the launcher's environment.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    bench.init_dist(w, torch.device("cpu"), backend="gloo", timeout_s=60)
    import torch.distributed as dist
    try:
        results[rank] = bench.max_over_ranks(values[rank], w, torch.device("cpu"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("values", [[3.5, 1.25], [0.5, 9.0]])
def test_max_over_ranks_with_two_gloo_ranks(values):
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, values, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert results[0] == results[1] == max(values)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(2.5, 1, torch.device("cpu")) == 2.5
    bench.init_dist(1, torch.device("cpu"), backend="gloo")  # no-op
