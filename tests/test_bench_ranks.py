"""The multi-rank side of bench.py on CPU (gloo, world size 2): timings are
combined as the maximum over ranks, and the reference arm runs on rank 0
only (the other ranks leave without work)."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.0], "cpu", world)
        # rank 1 returns from the reference arm at once (it would print nothing)
        if rank == 1:
            class A:  # the parsed arguments the reference arm reads
                layers, T, decode_batch, steps, warmup, gpus = 1, 64, 1, 1, 1, 2
            bench.run_reference(A, rank)
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_reference_arm_rank_gate():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert out[r] == [2.0, 10.0, 3.0]


def test_max_over_ranks_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1, 2.5], "cpu", 1) == [1.0, 2.5]
