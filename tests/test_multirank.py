"""The N > 1 path of bench.py on CPU: two gloo ranks, no GPU.

Every rank runs an independent replica (weak scaling, no data-path
collective); the only collectives are the barrier and the reduction of the
step time (max over ranks) and of the tokens (sum over ranks).
"""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ms = [3.0, 5.0, 4.0][rank]           # per-rank device step time
    out = bench.aggregate_over_ranks(ms, 8192.0, dist, torch.device("cpu"))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, out))


@pytest.mark.parametrize("world", [2, 3])
def test_two_rank_aggregation_is_max_time_and_total_tokens(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want_ms = max([3.0, 5.0, 4.0][:world])
    for r in range(world):
        ms, tok, val = res[r]
        assert ms == want_ms
        assert tok == 8192.0 * world
        assert abs(val - tok / (ms / 1e3)) < 1e-6


def test_single_rank_passthrough():
    import bench
    ms, tok, val = bench.aggregate_over_ranks(2.0, 100.0)
    assert (ms, tok) == (2.0, 100.0) and abs(val - 50000.0) < 1e-9
