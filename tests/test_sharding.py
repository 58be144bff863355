"""Row sharding of the layer stack on CPU: the partition of
rows / sequences over ranks, and that the pieces reproduce the whole stack
(query rows are independent given the prefix), checked with the oracle and
with two gloo ranks.  The GPU side of a shard is an ordinary stack call with
a row offset; no collective is on the data path."""
import os
import socket

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from lightning_indexer_top_relu_b200 import sharding, synth


@pytest.mark.parametrize("Lq", [1, 7, 512, 8192, 10000])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_zigzag_chunks_cover_every_row_once(Lq, world):
    rows = []
    for r in range(world):
        for i0, n in sharding.zigzag_chunks(Lq, world, r):
            assert n > 0 and (i0 % 128 == 0)
            rows.extend(range(i0, i0 + n))
    assert sorted(rows) == list(range(Lq))


@settings(max_examples=300, deadline=None)
@given(B=st.integers(1, 40), Lq=st.integers(1, 20000), world=st.integers(1, 16),
       align=st.sampled_from([1, 8, 64, 128]))
def test_shards_partition_the_rows_of_every_sequence(B, Lq, world, align):
    """Over all ranks every (sequence, row) pair is covered exactly once, each
    chunk lies inside the problem, and row chunks start on `align` rows."""
    seen = np.zeros((B, Lq), dtype=np.int32)
    for r in range(world):
        for ch in sharding.shard(B, Lq, world, r, align):
            assert ch.nb > 0 and ch.n > 0
            assert 0 <= ch.b0 and ch.b0 + ch.nb <= B and 0 <= ch.i0 and ch.i0 + ch.n <= Lq
            if B == 1:
                assert ch.i0 % align == 0
            seen[ch.b0:ch.b0 + ch.nb, ch.i0:ch.i0 + ch.n] += 1
    assert np.all(seen == 1)


@pytest.mark.parametrize("world", [2, 4, 8])
def test_zigzag_balances_the_causal_cost(world):
    Lq = 65536
    cost = [sum(sharding.chunk_cost(ch, 0) for ch in sharding.shard(1, Lq, world, r))
            for r in range(world)]
    assert max(cost) / (sum(cost) / world) <= 1.02
    # contiguous blocks instead give the last rank (2*world - 1) / world x the mean
    blk = [sum(t + 1 for t in range(r * Lq // world, (r + 1) * Lq // world)) for r in range(world)]
    assert max(blk) / (sum(blk) / world) > 1.45


def test_batches_split_by_sequence():
    chunks = [sharding.shard(32, 1, 3, r) for r in range(3)]
    assert [c[0].nb for c in chunks] == [11, 11, 10]
    assert [c[0].b0 for c in chunks] == [0, 11, 22]
    assert sharding.shard(2, 5, 4, 3) == []          # more ranks than sequences


def _full_and_sharded(world, align=64):
    wl = synth.WORKLOADS["tiny_prefill"]
    layers = synth.make_layers(wl)
    outs, idxs, _ = oracle.layer_stack(wl.pattern, layers, wl.k)
    parts = []
    for r in range(world):
        for ch in sharding.shard(wl.B, wl.Lq, world, r, align):
            o, ix, _ = oracle.layer_stack(wl.pattern, sharding.slice_layers(layers, ch), wl.k,
                                          q_offset=wl.q_offset + ch.i0)
            parts.append((r, ch, o, ix))
    return wl, outs, idxs, parts


@pytest.mark.parametrize("world", [2, 3])
def test_shards_reproduce_the_whole_stack(world):
    wl, outs, idxs, parts = _full_and_sharded(world)
    seen = np.zeros(wl.Lq, dtype=int)
    for _, ch, o, ix in parts:
        rows = slice(ch.i0, ch.i0 + ch.n)
        seen[rows] += 1
        for l in range(wl.n_layers):
            assert np.array_equal(ix[l], idxs[l][rows])          # same arithmetic per row
            assert np.array_equal(o[l], outs[l][rows])
    assert np.all(seen == 1)


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
    wl = synth.WORKLOADS["tiny_prefill"]
    layers = synth.make_layers(wl)
    # this rank's rows of the last layer, then one all-gather to assemble them
    mine = torch.full((wl.Lq, wl.Hq, wl.d), float("nan"), dtype=torch.float64)
    for ch in sharding.shard(wl.B, wl.Lq, world, rank, 64):
        o, _, _ = oracle.layer_stack(wl.pattern, sharding.slice_layers(layers, ch), wl.k,
                                     q_offset=ch.i0)
        mine[ch.i0: ch.i0 + ch.n] = torch.from_numpy(o[-1].reshape(ch.n, wl.Hq, wl.d))
    got = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(got, mine)
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        full = torch.full_like(mine, float("nan"))
        for g in got:
            have = ~torch.isnan(g[:, 0, 0])
            full[have] = g[have]
        ref, _, _ = oracle.layer_stack(wl.pattern, layers, wl.k)
        q.put(bool(torch.equal(full, torch.from_numpy(ref[-1].reshape(wl.Lq, wl.Hq, wl.d)))))


def test_two_gloo_ranks_assemble_the_whole_stack():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    ok = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert ok
