"""Drift-triggered refresh and row sharding on the GPU.

Both are compositions of entry points that have their own parity tests (the
layer stack, indexer, top-k, the stack's attention step, the overlap
kernel); these tests check the plumbing around them:

* DriftRefreshStack over GpuBackend takes the same refresh decisions as over
  the CPU oracle backend, its probe overlaps agree with the oracle's, and its
  outputs equal a static GPU stack of the pattern it chose;
* the shards of one stack (zig-zag row chunks, each an ordinary stack call
  with a row offset), run one after another on this GPU, reassemble the
  whole stack's index rows bit for bit and its outputs within the attention
  tolerance.
"""
import numpy as np
import pytest
import torch

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


@pytest.mark.parametrize("replace,tau", [((), 0.5), ((2,), 0.5), ((), 1.0)])
def test_drift_refresh_on_the_gpu_matches_the_oracle_policy(ic, replace, tau):
    layers = _layers(replace)
    cpu = DriftRefreshStack(WL.pattern, OracleBackend(layers, WL.k), WL.k, tau, 128)
    cpu.forward()
    cuda = [{n: t.cuda() for n, t in L.items()} for L in layers]
    gpu = DriftRefreshStack(WL.pattern, GpuBackend(cuda, _dims(ic)), WL.k, tau, 128)
    outs = gpu.forward()
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    assert gpu.run_pattern == cpu.run_pattern
    for a, b in zip(gpu.overlaps, cpu.overlaps):
        assert (a is None) == (b is None)
        if a is not None:
            assert abs(a - b) <= 0.02, (gpu.overlaps, cpu.overlaps)
    # the same outputs as a static stack of the chosen pattern
    ref = ic.LayerStack(gpu.run_pattern, cuda, _dims(ic))
    ref.forward()
    torch.cuda.synchronize()
    for l in range(WL.n_layers):
        assert (outs[l].float() - ref.outs[l].float()).abs().max().item() <= ATTN_ATOL


@pytest.mark.parametrize("world", [2, 3])
def test_shards_run_in_turn_reassemble_the_whole_stack(ic, world):
    layers = [{n: t.cuda() for n, t in L.items()} for L in _layers()]
    dims = _dims(ic)
    whole = ic.LayerStack(WL.pattern, layers, dims, dump_idx=True)
    whole.forward()
    torch.cuda.synchronize()
    seen = np.zeros(WL.Lq, dtype=np.int32)
    for rank in range(world):
        part = sharding.ShardedStack(WL.pattern, layers, dims, world, rank, dump_idx=True)
        part.forward()
        torch.cuda.synchronize()
        assert ic.get_last_device_error() == 0
        for ch, st in zip(part.chunks, part.stacks):
            rows = slice(ch.i0, ch.i0 + ch.n)
            seen[rows] += 1
            for l in range(WL.n_layers):
                assert torch.equal(st.dumps[l][0], whole.dumps[l][0, rows])
                err = (st.outs[l][0].float() - whole.outs[l][0, rows].float()).abs().max().item()
                assert err <= ATTN_ATOL
    assert np.all(seen == 1)
