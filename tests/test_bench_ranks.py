"""bench.py's multi-rank host logic on CPU: two gloo ranks (one process per
rank, as torchrun launches them) agree on the max-over-ranks timing, get
different inputs of the same shape, and only rank 0 produces the reference
arm's line."""
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
                      WORLD_SIZE=str(world))
    import bench
    from synthetic import get_workload
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        per_rank = [10.0 + rank, 100.0 - rank]
        mx = bench.max_over_ranks(per_rank, world)
        wl = bench.rank_workload(get_workload("768p"), rank)

        class A:
            workload, steps, warmup, cpu_rows = "tiny", 1, 3, 8
        ref = bench.run_reference(A, rank, world) if rank != 0 else "skip"
        out.put((rank, mx, wl.seed, (wl.B, wl.H, wl.T, wl.N), ref))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, mx0, seed0, shape0, _), (r1, mx1, seed1, shape1, ref1) = res
    assert mx0 == mx1 == [11.0, 100.0]
    assert seed0 != seed1 and shape0 == shape1
    assert ref1 is None          # the reference arm runs on rank 0 only
