"""The multi-GPU bench path on CPU: two gloo ranks, each timing its own
independent block; the job time is the slowest rank's and every rank sees
the same value (no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, _ = bench.dist_init()
    try:
        t = bench.dist_max(10.0 + 5.0 * r, w)
        bench.dist_barrier(w)
        q.put((r, w, t, bench.rank_seed_offset(r)))
    finally:
        bench.dist_done(w)


def test_two_gloo_ranks_max_timing_and_distinct_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [r[:3] for r in res] == [(0, 2, 15.0), (1, 2, 15.0)]
    assert res[0][3] != res[1][3]            # each rank draws its own block
