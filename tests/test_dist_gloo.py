"""The multi-process plumbing with world size 2 on gloo (CPU): sharding of
independent shape pairs, barrier, and the max-over-ranks timing reduction."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from spatial_spectral_attention_b200 import dist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    w, r, _ = dist.init("gloo", timeout_s=30)
    mine = dist.shard(7, w, r)
    dist.barrier(w)
    m = dist.max_over_ranks(10.0 + r, w, device="cpu")
    q.put((r, mine, m))
    dist.finalize(w)


def test_shard_covers_items_once():
    for n in (1, 5, 8, 13):
        for ws in (1, 2, 3, 8):
            got = [i for r in range(ws) for i in dist.shard(n, ws, r)]
            assert got == list(range(n))


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][1] + res[1][1] == list(range(7))
    assert res[0][2] == res[1][2] == 11.0
