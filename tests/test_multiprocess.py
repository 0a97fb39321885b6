"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The library shards with no exchange: each rank decodes its own sequence and the
job's time is the slowest rank's.  These tests run the host side of that on two
CPU processes: the max-over-ranks reduction, distinct per-rank inputs, and the
reference arm doing no work on ranks other than 0.
"""

import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import numpy as np

    import bench
    from decode_attention_13_b200 import synth

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # the job's time is the slowest rank's
        t = bench.max_over_ranks(1.5 + rank, world)
        # every rank draws its own sequence
        lay = synth.layer(bench.rank_seed(1, rank, 0), 1, 1, 1, 16, dtype=np.float32)
        k = torch.from_numpy(lay["k"].astype(np.float64)).reshape(-1)
        ks = [torch.zeros_like(k) for _ in range(world)]
        dist.all_gather(ks, k)
        distinct = not torch.equal(ks[0], ks[1])
        # the reference arm: ranks other than 0 return without work or output
        import contextlib
        import io

        class A:
            config, steps, warmup, cpu_seconds = 0, 1, 0, 0.05

        buf = io.StringIO()
        if rank != 0:
            with contextlib.redirect_stdout(buf):
                bench.run_reference(A(), rank, world)
        q.put((rank, t, distinct, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_rank_host_logic():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]          # max over ranks on every rank
    assert all(r[2] for r in res)                     # independent per-rank inputs
    assert res[1][3] == ""                            # rank 1 of the reference arm: no work
