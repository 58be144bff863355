"""Drift-triggered refresh and row sharding on the GPU.

Both are compositions of entry points that have their own parity tests (the
layer stack, indexer, top-k, the stack's attention step, the overlap
kernel); these tests check the plumbing around them:

* DriftRefreshStack over GpuBackend takes the same refresh decisions as over
  the CPU oracle backend, on the default stream and on a stream of its own;
  its probe overlaps agree with the oracle's, and its outputs match the
  oracle's stack of the pattern it chose (top-k overlap >= 0.99, attention
  within 2e-2 on rows whose index sets agree);
* the shards of one stack (zig-zag row chunks of one sequence, or whole
  sequences of a batch; each an ordinary stack call with a row offset), run
  one after another on this GPU, match the oracle's stack computed on that
  shard's slice of the inputs, and reassemble the whole GPU stack's index
  rows bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from lightning_indexer_top_relu_b200 import build, sharding, synth
from lightning_indexer_top_relu_b200.drift import DriftRefreshStack, GpuBackend
from test_drift import OracleBackend

pytestmark = pytest.mark.gpu

ATTN_ATOL = 2e-2
# 700 rows, k = 64: rows t < 512 attend dense-masked, the rest gather
WL = synth.Workload("drift_gpu", 1, 700, 700, 4, 32, 128, 64, 16, 128, "FSSS", 0, 43, True)


@pytest.fixture(scope="module")
def ic():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    from lightning_indexer_top_relu_b200 import indexcache
    return indexcache


def _layers(replace=()):
    layers = synth.make_layers(WL)
    other = synth.make_layers(synth.custom(Lq=WL.Lq, n_layers=WL.n_layers, H_I=WL.H_I,
                                           d_I=WL.d_I, k=WL.k, Hq=WL.Hq, d=WL.d, cfg_id=44))
    for l in replace:
        for n in ("q_idx", "k_idx", "w"):
            layers[l][n] = other[l][n]
    return layers


def _dims(ic, wl=WL):
    return ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)


def _overlap(a, b):
    return np.array([len(set(x[x >= 0].tolist()) & set(y[y >= 0].tolist())) / max(1, (y >= 0).sum())
                     for x, y in zip(a, b)])


def _match_oracle(pattern, cpu_layers, k, q_offset, dumps, outs, Hq, d):
    """GPU index rows and outputs of a stack against the oracle's stack on the
    same inputs: mean top-k overlap >= 0.99 per layer, attention within the
    tolerance on the rows whose index sets agree exactly."""
    o_outs, o_idxs, _ = oracle.layer_stack(pattern, cpu_layers, k, q_offset)
    for l in range(len(pattern)):
        g = dumps[l].cpu().numpy().reshape(-1, k)
        ov = _overlap(g, o_idxs[l])
        assert ov.mean() >= 0.99, (l, ov.mean(), ov.min())
        same = np.array([np.array_equal(a, b) for a, b in zip(g, o_idxs[l])])
        assert same.mean() >= 0.9, (l, same.mean())
        got = outs[l].float().cpu().numpy().reshape(-1, Hq, d)
        assert np.abs(got[same] - o_outs[l][same]).max() <= ATTN_ATOL


@pytest.mark.parametrize("own_stream", [False, True])
@pytest.mark.parametrize("replace,tau", [((), 0.5), ((2,), 0.5), ((), 1.0)])
def test_drift_refresh_on_the_gpu_matches_the_oracle_policy(ic, replace, tau, own_stream):
    layers = _layers(replace)
    cpu = DriftRefreshStack(WL.pattern, OracleBackend(layers, WL.k), WL.k, tau, 128)
    cpu.forward()
    cuda = [{n: t.cuda() for n, t in L.items()} for L in layers]
    torch.cuda.synchronize()
    stream = torch.cuda.Stream() if own_stream else None
    gpu = DriftRefreshStack(WL.pattern, GpuBackend(cuda, _dims(ic), stream=stream), WL.k, tau, 128)
    outs = gpu.forward()
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    assert gpu.run_pattern == cpu.run_pattern
    for a, b in zip(gpu.overlaps, cpu.overlaps):
        assert (a is None) == (b is None)
        if a is not None:
            assert abs(a - b) <= 0.02, (gpu.overlaps, cpu.overlaps)
    # a static GPU stack of the chosen pattern gives the same outputs, and its
    # index rows and outputs match the oracle's stack of that pattern
    ref = ic.LayerStack(gpu.run_pattern, cuda, _dims(ic), dump_idx=True)
    ref.forward()
    torch.cuda.synchronize()
    for l in range(WL.n_layers):
        assert (outs[l].float() - ref.outs[l].float()).abs().max().item() <= ATTN_ATOL
    _match_oracle(gpu.run_pattern, layers, WL.k, 0, ref.dumps, outs, WL.Hq, WL.d)


SHARD_B3 = synth.Workload("shard_b3", 3, 300, 300, 2, 32, 128, 64, 16, 128, "FS", 0, 45, True)


@pytest.mark.parametrize("wl,world", [(WL, 2), (WL, 3), (SHARD_B3, 2)])
def test_shards_run_in_turn_match_the_oracle_and_the_whole_stack(ic, wl, world):
    cpu_layers = synth.make_layers(wl) if wl is not WL else _layers()
    layers = [{n: t.cuda() for n, t in L.items()} for L in cpu_layers]
    dims = _dims(ic, wl)
    whole = ic.LayerStack(wl.pattern, layers, dims, dump_idx=True)
    whole.forward()
    torch.cuda.synchronize()
    seen = np.zeros((wl.B, wl.Lq), dtype=np.int32)
    for rank in range(world):
        part = sharding.ShardedStack(wl.pattern, layers, dims, world, rank, dump_idx=True)
        part.forward()
        torch.cuda.synchronize()
        assert ic.get_last_device_error() == 0
        for ch, st in zip(part.chunks, part.stacks):
            bs, rows = slice(ch.b0, ch.b0 + ch.nb), slice(ch.i0, ch.i0 + ch.n)
            seen[bs, rows] += 1
            # each shard against the oracle on the shard's own slice of the inputs
            _match_oracle(wl.pattern, sharding.slice_layers(cpu_layers, ch), wl.k,
                          wl.q_offset + ch.i0, st.dumps, st.outs, wl.Hq, wl.d)
            for l in range(wl.n_layers):
                assert torch.equal(st.dumps[l], whole.dumps[l][bs, rows])
    assert np.all(seen == 1)
