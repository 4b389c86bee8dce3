"""The multi-rank host logic of bench.py on CPU (gloo, world size 2): the
timing reduction takes the maximum over ranks, and only rank 0 runs the
reference arm.  The data path itself has no cross-rank exchange (replicas)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws),
                      LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(10.0 + 3.0 * rank, ws)
        env = bench.dist_init()

        class A:
            steps, warmup = 1, 0
        # rank != 0 returns immediately from the reference arm, with no work
        ref_rc = bench.run_reference(A(), ws, rank) if rank != 0 else 0
        dist.barrier()
        q.put((rank, got, env, ref_rc))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_reference_rank_gating():
    ws = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(ws))
    for rank, got, env, ref_rc in res:
        assert got == 13.0                      # max of 10 and 13
        assert env == (ws, rank, rank)
        assert ref_rc == 0


def test_single_rank_max_is_identity():
    import bench
    assert bench.max_over_ranks(4.5, 1) == 4.5
