"""bench.py's multi-rank plumbing on CPU: two gloo ranks, max-over-ranks timing
and one independent problem per rank (weak scaling, no data-path collective)."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import bench
    from long_context_attention_bifocal_b200 import workloads as W
    t = bench.max_over_ranks(10.0 + rank, world)
    bench.barrier(world)
    seed = bench.rank_seed(5, rank)
    qd, _, _ = W.decode_inputs(1, 4, 2, 8, 16, seed=seed)
    q.put((rank, t, qd.float().sum().item()))
    torch.distributed.destroy_process_group()


def test_two_gloo_ranks():
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
    assert [r[1] for r in res] == [11.0, 11.0]  # both ranks see the slowest time
    assert res[0][2] != res[1][2]               # independent problems per rank
