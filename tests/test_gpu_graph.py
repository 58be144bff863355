"""The layer stack captured into a CUDA graph and replayed, and two stacks
running at once on two streams, through the C ABI.

ic_layer_stack_forward enqueues kernels (and, for decode rows, cluster
launches) on the caller's stream without any host synchronisation, so a
forward can be captured once and replayed.  A replay must give the eager
run's outputs and index rows bit for bit, and it must read the input
buffers at replay time: after new values are written into the captured
tensors, a replay equals an eager run over the new values.
"""
import pytest
import torch

from lightning_indexer_top_relu_b200 import build, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ic():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    from lightning_indexer_top_relu_b200 import indexcache
    return indexcache


CASES = [
    # name, B, Lq, Lk, q_offset, k, pattern
    ("decode_clusters", 40, 1, 3000, 2999, 2048, "FSSF"),     # splits merged in clusters
    ("decode_workspace", 4, 1, 3000, 2999, 2048, "FSSS"),     # split partials + combine kernel
    ("prefill_dense_and_gather", 1, 700, 700, 0, 64, "FSFS"),  # dense-masked and gathered rows
]


def _eager(ic, st, stream):
    with torch.cuda.stream(stream):
        st.forward(stream)
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    return [o.clone() for o in st.outs], [d.clone() for d in st.dumps]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_graph_replay_equals_eager_run(ic, case):
    name, B, Lq, Lk, q0, k, pattern = case
    wl = synth.custom(B=B, Lq=Lq, Lk=Lk, q_offset=q0, n_layers=len(pattern), H_I=64, d_I=128, k=k,
                      Hq=16, d=128, pattern=pattern, cfg_id=62)
    layers = [{n: t.cuda() for n, t in L.items()} for L in synth.make_layers(wl)]
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    st = ic.LayerStack(pattern, layers, dims, want_lse=True, dump_idx=True)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    outs, dumps = _eager(ic, st, side)            # the first call sets the library up

    for o in st.outs:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st.forward()
    g.replay()
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    for l in range(len(pattern)):
        assert torch.equal(st.outs[l], outs[l]), (name, l)
        assert torch.equal(st.dumps[l], dumps[l]), (name, l)

    # new inputs written into the captured tensors: the replay reads them
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    for L in layers:
        for key in ("q", "q_idx"):
            L[key].copy_(torch.randn(L[key].shape, generator=gen, device="cuda",
                                     dtype=torch.float32).to(L[key].dtype) / 8)
    g.replay()
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    replayed = [o.clone() for o in st.outs], [d.clone() for d in st.dumps]
    fresh = _eager(ic, st, side)
    for l in range(len(pattern)):
        assert torch.equal(replayed[0][l], fresh[0][l]), (name, l)
        assert torch.equal(replayed[1][l], fresh[1][l]), (name, l)
    assert not all(torch.equal(a, b) for a, b in zip(fresh[0], outs))
    del g


def test_two_stacks_on_two_streams_run_independently(ic):
    """The library keeps no state from one call to the next: two stacks over
    different inputs, enqueued on two streams without synchronising in
    between (so their kernels may overlap), each give their own sequential
    results bit for bit."""
    runs = []
    for cfg, pattern in ((63, "FSFS"), (64, "FFSS")):
        wl = synth.custom(B=2, Lq=300, Lk=1300, q_offset=1000, n_layers=4, H_I=32, d_I=128, k=256,
                          Hq=16, d=128, pattern=pattern, cfg_id=cfg)
        layers = [{n: t.cuda() for n, t in L.items()} for L in synth.make_layers(wl)]
        dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
        runs.append(ic.LayerStack(pattern, layers, dims, want_lse=True, dump_idx=True))
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())     # inputs and workspaces are ready
    alone = [_eager(ic, st, s) for st, s in zip(runs, streams)]
    for st in runs:
        for o in st.outs:
            o.zero_()
    torch.cuda.synchronize()
    for _ in range(3):                       # several overlapping rounds
        for st, s in zip(runs, streams):
            with torch.cuda.stream(s):
                st.forward(s)
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    for st, (outs, dumps) in zip(runs, alone):
        for l in range(4):
            assert torch.equal(st.outs[l], outs[l])
            assert torch.equal(st.dumps[l], dumps[l])
