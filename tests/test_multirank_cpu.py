"""Host-side logic of the multi-GPU run, on CPU with two gloo ranks: every rank gets its own
batch shard (same per-GPU shape, its own seed: weak scaling, no data exchange), and the step
time reported is the maximum over ranks.  The attention path itself has no collective: every
(b, h) slice is independent."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import datetime
    import bench
    import workloads
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        s = bench.shard_shape(workloads.TINY, r)
        d = workloads.make_layer(s)
        t = 1.5 + r                       # a per-rank "step time"
        mx = bench.reduce_max(t)
        q.put((r, w, local, s.seed, workloads.sha256_of(d), mx, bench.flops_per_step(s)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, l0, seed0, h0, m0, f0), (r1, w1, l1, seed1, h1, m1, f1) = res
    assert (r0, r1, w0, w1, l0, l1) == (0, 1, 2, 2, 0, 1)
    assert seed0 != seed1 and h0 != h1          # each rank draws its own shard
    assert m0 == m1 == 2.5                      # max over ranks, identical on every rank
    assert f0 == f1                             # same per-GPU work: weak scaling


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.25) == 3.25
