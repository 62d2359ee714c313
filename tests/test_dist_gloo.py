"""Multi-rank host logic on CPU (gloo, world size 2): sharding of independent
sequences, the barrier, and the max-over-ranks time that bench.py reports."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from recurrent_vision_backbone_key_b200 import dist as rdist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, w = rdist.init_from_env(backend="gloo", timeout_s=30)
    rdist.barrier()
    mx = rdist.max_over_ranks(10.0 + r)
    sm = rdist.sum_over_ranks(1.0)
    q.put((r, w, mx, sm, rdist.shard(384, r, w)))
    rdist.finalize()


def test_shard_covers_every_unit_once():
    for n in (0, 1, 7, 384, 1000):
        for world in (1, 2, 3, 8):
            spans = [rdist.shard(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def test_gloo_two_ranks():
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
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 for r in res)
    assert all(r[2] == 11.0 for r in res)
    assert all(r[3] == 2.0 for r in res)
    assert res[0][4] == (0, 192) and res[1][4] == (192, 384)
