"""Multi-rank host logic of the benchmark on CPU: two gloo ranks, no GPU.

Rows are independent, so ranks share nothing on the data path: each takes its own rows and
the job's time is the slowest rank's. These tests run the benchmark's own helpers under a
real two-process group.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from structured_compressed_linear_b200.workloads import WORKLOADS, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank timings: the reduction must give every rank the element-wise max
        mine = torch.tensor([1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)], dtype=torch.float64)
        got = bench.max_over_ranks(mine.clone(), world)
        # per-rank rows of a small layer
        L = WORKLOADS[1][0].with_M(64)
        X, _ = make_inputs(L)
        Xr = bench.rank_rows(X, rank)
        gathered = [torch.empty_like(Xr) for _ in range(world)]
        dist.all_gather(gathered, Xr)
        if rank == 0:
            out.put((got.tolist(), [g.clone() for g in gathered], X.clone()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_timings_are_max_over_ranks(two_ranks):
    got, _, _ = two_ranks
    assert got == [2.0, 5.0, 0.5]


def test_ranks_take_distinct_permutations_of_the_rows(two_ranks):
    _, gathered, X = two_ranks
    r0, r1 = gathered
    assert torch.equal(r0, X)                       # rank 0 keeps the seeded rows
    assert not torch.equal(r1, r0)                  # rank 1 gets other rows ...
    key = lambda t: sorted(map(tuple, t.float().tolist()))
    assert key(r1) == key(r0)                       # ... a permutation of the same ones


def test_whole_job_value_counts_every_rank():
    # 2 ranks x 1 TFLOP of dense work in 1 s of the slowest rank = 2 TFLOP/s
    assert bench.whole_job_value(1e12, 1000.0, 2) == pytest.approx(2.0)
    assert bench.whole_job_value(1e12, 500.0, 1) == pytest.approx(2.0)


def test_reference_arm_is_rank_zero_only(capsys):
    layers = WORKLOADS[1]

    class A:
        steps, warmup = 1, 0

    bench.run_reference(A, layers, 1, rank=1, world=2)
    assert capsys.readouterr().out == ""
