"""Cross-layer index overlap on the GPU against the oracle
(integer results: bit-exact), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from lightning_indexer_top_relu_b200 import build, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ic():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    from lightning_indexer_top_relu_b200 import indexcache
    return indexcache


@pytest.mark.parametrize("n,k,Lk", [(1, 1, 1), (300, 24, 60), (1000, 2048, 8192),
                                    (37, 100, 262144)])
def test_overlap_random_rows_match_oracle(ic, n, k, Lk):
    rng = np.random.default_rng(n + k)
    a = rng.integers(-1, Lk, size=(n, k)).astype(np.int32)      # holes, repeats, any order
    b = a.copy()
    flip = rng.random(a.shape) < 0.3
    b[flip] = rng.integers(-1, Lk, size=int(flip.sum()))
    ref = oracle.index_overlap(a, b, Lk)
    got = ic.index_overlap(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), Lk)
    assert ic.get_last_device_error() == 0
    assert np.array_equal(got.cpu().numpy(), ref)


def test_overlap_bad_entries_are_skipped_and_reported(ic):
    a = np.array([[0, 5, 9, -1], [1, 2, 3, 4]], dtype=np.int32)
    b = np.array([[5, 10, -7, 0], [4, 3, 2, 1]], dtype=np.int32)   # 10 and -7 are invalid for Lk=10
    got = ic.index_overlap(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), 10)
    assert ic.get_last_device_error() == 1                          # IC_ERR_INVALID_ARG
    assert got.cpu().numpy().tolist() == [[2, 3, 2], [4, 4, 4]]
    assert ic.get_last_device_error() == 0


def test_overlap_of_two_full_layers_at_8k(ic):
    """The benchmarked 8K workload: the two F layers' index caches from the
    stack, every row against the oracle, and the overlap in the band the
    pages report for adjacent layers of real models."""
    wl = synth.WORKLOADS["prefill_8k"]
    layers = synth.make_layers(wl, indexer_for_all=False)
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    cuda = [{n: t.cuda() for n, t in L.items()} for L in layers]
    st = ic.LayerStack(wl.pattern, cuda, dims, dump_idx=True)
    st.forward()
    torch.cuda.synchronize()
    f = [l for l, c in enumerate(wl.pattern) if c == "F"]
    a, b = st.dumps[f[0]], st.dumps[f[1]]
    got = ic.index_overlap(a, b, wl.Lk).cpu().numpy()
    ref = oracle.index_overlap(a.cpu().numpy().reshape(-1, wl.k), b.cpu().numpy().reshape(-1, wl.k),
                               wl.Lk)
    assert ic.get_last_device_error() == 0
    assert np.array_equal(got, ref)
    rows = np.arange(wl.k, wl.Lq)                  # rows whose sets are a real choice (t >= k)
    ov = oracle.overlap_fraction(got[rows], wl.k)
    assert 0.5 <= ov.mean() <= 1.0
