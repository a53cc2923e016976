"""The N > 1 host path of bench.py on CPU: world size 2 over gloo.

The NVFP4 path shards by rows with no exchange step, so the multi-GPU bench runs independent replicas;
what needs checking is the plumbing: rank set-up from the torchrun environment, the barrier, the
max-over-ranks timing, and that only rank 0 runs the reference arm.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    ws, r, local = bench.dist_init("gloo")
    bench.barrier(ws)
    # each rank reports a different elapsed time; every rank must see the maximum
    got = bench.max_over_ranks(10.0 + 5.0 * r, ws)

    class Args:
        steps, warmup = 1, 0
    ref = bench.run_reference(Args(), ws, r) if r != 0 else "rank0-skipped"
    bench.barrier(ws)
    dist.destroy_process_group()
    q.put((r, ws, local, got, ref))


def test_replicas_plumbing_world_size_2():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for r, (rank, ws, local, got, ref) in enumerate(res):
        assert (rank, ws, local) == (r, world, r)
        assert got == 15.0
    assert res[1][4] is None          # non-zero ranks do no reference work and print nothing
