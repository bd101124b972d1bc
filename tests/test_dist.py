"""Multi-rank plumbing on CPU (gloo, world size 2): unit sharding covers every
unit exactly once, and a step's time is the maximum over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from oracle_top_kv_b200 import dist as hdist


def test_units_for_rank_partitions_exactly():
    for n in (0, 1, 7, 16, 128):
        for w in (1, 2, 3, 8):
            seen = []
            for r in range(w):
                seen += list(hdist.units_for_rank(n, r, w))
            assert seen == list(range(n))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    hdist.init("gloo", timeout_s=60)
    r, w, _ = hdist.world()
    mine = list(hdist.units_for_rank(16, r, w))
    hdist.barrier()
    slowest = hdist.max_over_ranks(10.0 + r)  # rank 1 is slower
    out.put((r, mine, slowest))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_rank_gloo_timing_and_sharding():
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
    assert [r for r, _, _ in res] == [0, 1]
    assert res[0][1] + res[1][1] == list(range(16))
    assert all(s == 11.0 for _, _, s in res)
