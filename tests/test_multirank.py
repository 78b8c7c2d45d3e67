"""The multi-rank plumbing of bench.py on CPU with the gloo backend,
world size 2: ranks take disjoint sequences of the workload recipe (weak
scaling, no data-path collective), and the reported time is the max over
ranks."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.workload("1m")
        off = bench.shard_offset(rank, w.B)
        seqs = list(range(off, off + w.B))
        # each rank's first raw keys come from its own sequences
        first = w.raw_keys_np(off, 0, 4).tolist()
        t = bench.max_over_ranks(float(10 + rank * 5), world, torch.device("cpu"))
        bench.barrier(world)
        q.put((rank, seqs, first, t))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_time_max():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (r0, s0, f0, t0), (r1, s1, f1, t1) = res
    assert set(s0).isdisjoint(s1) and sorted(s0 + s1) == list(range(8))
    assert f0 != f1  # different sequences, different keys
    assert t0 == t1 == 15.0  # both ranks report the slowest rank's time
