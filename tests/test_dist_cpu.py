"""The bench's multi-rank host logic on CPU: two gloo ranks (no GPU).

Each rank runs its own call (replicas, no data-path collective); the only
cross-rank steps are the barrier around the timed region and the max over
ranks of the measured times. Both are exercised here with world size 2.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench._barrier(dist)
    mine = 3.0 + rank * 1.5          # per-rank device time (ms)
    got = bench._max_over_ranks(dist, mine)
    bench._barrier(dist)
    q.put((rank, got))
    dist.destroy_process_group()


def test_two_rank_max_and_barrier():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 4.5, 1: 4.5}


def test_single_rank_is_identity():
    import bench
    assert bench._max_over_ranks(None, 2.5) == 2.5


def test_traffic_hash_ignores_comments_but_not_code():
    import bench
    a = 'int a; // note\n/* block */ asm("x // y"); int  b;\n'
    b = 'int a;\n asm("x // y");    int b; // another note\n'
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(a.replace("int  b", "int c"))
    assert bench._code_only(a) != bench._code_only(a.replace("x // y", "x / y"))   # strings are code
