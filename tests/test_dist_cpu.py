"""The bench's multi-rank host logic on CPU: two gloo ranks (no GPU).

The heads of one call are split across the ranks (no data-path collective);
the only cross-rank steps are the barrier around the timed region, the max
over ranks of the measured times and sums of per-rank counts. All are
exercised here with world size 2, together with the head partition.
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


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import workloads
    w0 = workloads.get("ragged_pe")                       # B=2, H=3: an uneven split over 2 ranks
    w, heads = bench.shard(w0, rank, world)
    Q, K, V = bench.shard_qkv(w0, heads)
    full = workloads.batch_qkv(w0)
    same = all(torch.equal(x, f[:, heads]) for x, f in zip((Q, K, V), full))
    got = [None] * world
    dist.all_gather_object(got, heads)
    total = bench._sum_over_ranks(dist, float(w.H))
    q.put((rank, same, got, total, w.H))
    dist.destroy_process_group()


def test_two_rank_head_split_covers_every_head_once():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = {r: (same, got, total, h) for r, same, got, total, h in (q.get(timeout=5) for _ in range(2))}
    for r in range(2):
        same, got, total, h = res[r]
        assert same                                      # a rank's heads are the full call's heads
        assert got == [[0, 1], [2]] and total == 3.0
    assert res[0][3] == 2 and res[1][3] == 1


def test_head_range_partitions():
    import bench
    for H in (1, 2, 5, 12, 40):
        for world in (1, 2, 3, 4, 8):
            parts = [bench.head_range(H, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == H
            assert all(parts[r][1] == parts[r + 1][0] for r in range(world - 1))
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
    assert [bench.head_range(40, r, 8) for r in range(8)] == [(5 * r, 5 * r + 5) for r in range(8)]


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
