"""bench.py's multi-rank host logic on CPU: world size 2 over gloo at 127.0.0.1.

With N GPUs every rank runs its own replica (the path has no exchange step); the ranks meet
only in barriers and in the max-over-ranks of the step time, and the reference arm runs on
rank 0 alone. These are the pieces exercised here, with the gloo backend standing in for NCCL.
"""
import datetime
import os
import socket
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=ws,
                                         timeout=datetime.timedelta(seconds=60))
    import bench

    bench.barrier(ws)
    step_ms = bench.max_over_ranks(1.5 + rank, ws, torch.device("cpu"))

    class A:   # the reference arm's arguments; rank 1 must return before touching them
        workload = "no-such-workload"
        steps = warmup = 1

    ref = "skipped"
    if rank == 1:
        bench.reference_arm(A, ws, rank)
        ref = "returned"
    bench.barrier(ws)
    torch.distributed.destroy_process_group()
    q.put((rank, step_ms, ref))


def test_two_ranks_barrier_and_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res == [(0, 2.5, "skipped"), (1, 2.5, "returned")], res
