"""The layer stack's fused indexer -> top-k on the GPU, through the C ABI.

On the fused path the F layer's score matrix is never stored: a sampled pass
sets per-row thresholds, the indexer keeps only candidates above them, an
exact selection runs on the candidates, and rows whose candidates do not
certify the result fall back to the plain indexer + top-k.  Whatever the
thresholds do, the index rows must be exactly the top-k of the scores the
GPU's indexer computes (ic_indexer_scores), so every test compares them bit
for bit with the oracle's sort-based top-k run on those very scores (the
parity rule for the top-k: bit-exact on the same score tensor), and with the
unfused stack (index rows and attention outputs identical).

Cases: ragged and multi-tile shapes, B > 1 with a continuation chunk, the
largest k the fused path takes (4096), the benchmarked 8K prefill, the long rows falling back (w = 0: all scores tie
at 0, the closed form [0 .. k-1]), about half the rows falling back (a tiny
threshold margin), and small workspaces that split the rows into chunks with
several fallback rounds each.
"""
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


def _dims(ic, wl):
    return ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)


def _stack(ic, wl, layers, fused, z=0.0, rows_per_chunk=0, pattern=None):
    st = ic.LayerStack(pattern or wl.pattern, layers, _dims(ic, wl), dump_idx=True,
                       fused_topk=fused, z=z, rows_per_chunk=rows_per_chunk)
    st.forward()
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    return st


def _expected(ic, wl, L, rows=None):
    """The oracle's top-k of the GPU's own indexer scores (rows: flattened
    row numbers, None = all)."""
    sc = ic.indexer_scores(L["q_idx"], L["k_idx"], L["w"], wl.q_offset)
    torch.cuda.synchronize()
    s = sc.reshape(-1, wl.Lk)
    if rows is not None:
        s = s[torch.as_tensor(rows, device=s.device)]
    tpos = oracle.row_positions(wl.B, wl.Lq, wl.q_offset, rows)
    return oracle.topk_sort(s.cpu().numpy(), tpos, wl.k)


def _blocks_with_long_rows(wl, QB, cap):
    """Query blocks holding a row with more than cap visible positions."""
    n = 0
    for b in range(wl.B):
        for i0 in range(0, wl.Lq, QB):
            t_last = wl.q_offset + min(wl.Lq, i0 + QB) - 1
            n += (min(t_last + 1, wl.Lk) > cap)
    return n


CASES = [
    # name, B, Lq, Lk, q_offset, H_I, d_I, k, Hq, d
    ("ragged_small", 1, 1000, 1000, 0, 4, 64, 64, 8, 64),
    ("eight_k_k512", 1, 8192, 8192, 0, 32, 128, 512, 16, 128),
    ("batch2_continuation", 2, 1500, 6000, 4500, 64, 128, 256, 16, 128),
    ("heads128", 1, 3000, 3000, 0, 128, 64, 128, 8, 64),
    # the largest k the fused path takes (4096): rows t >= 10000 see more
    # than twice the 4k-entry list, so they run on sampled thresholds
    ("max_k_continuation", 1, 2000, 12000, 10000, 16, 128, 4096, 8, 64),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_fused_rows_equal_topk_of_gpu_scores_and_unfused_stack(ic, case):
    name, B, Lq, Lk, q0, H_I, d_I, k, Hq, d = case
    wl = synth.Workload(name, B, Lq, Lk, 2, H_I, d_I, k, Hq, d, "FS", q0, 51, True)
    layers = [{n: t.cuda() for n, t in L.items()} for L in synth.make_layers(wl)]
    fused = _stack(ic, wl, layers, 1)
    plain = _stack(ic, wl, layers, 0)
    want = _expected(ic, wl, layers[0])
    got = fused.dumps[0].cpu().numpy().reshape(-1, k)
    bad = np.nonzero(~np.all(got == want, axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[:5]}"
    for l in range(2):
        assert torch.equal(fused.dumps[l], plain.dumps[l])
        assert torch.equal(fused.outs[l], plain.outs[l])


def test_fused_selection_cuts_ties_at_the_kth_score(ic):
    """300 positions share one (scaled) key vector, so every query scores
    them equally, and where that score is positive they are a row's top
    scores: rows that see more of them than k keep only the lowest
    positions of the tie (the exact selection's tie cut).  Index rows equal
    the oracle's sort of the GPU's own scores, fused or not."""
    wl = synth.Workload("tie_cut", 1, 3000, 3000, 2, 8, 64, 128, 8, 64, "FS", 0, 53, True)
    layers = [{n: t.cuda() for n, t in L.items()} for L in synth.make_layers(wl)]
    tied = torch.arange(7, 3000, 10, device="cuda")                    # 300 positions
    kk = layers[0]["k_idx"]
    kk[0, tied] = (8.0 * kk[0, 7].float()).to(kk.dtype)
    fused = _stack(ic, wl, layers, 1)
    plain = _stack(ic, wl, layers, 0)
    want = _expected(ic, wl, layers[0])
    got = fused.dumps[0].cpu().numpy().reshape(-1, wl.k)
    bad = np.nonzero(~np.all(got == want, axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[:5]}"
    assert torch.equal(fused.dumps[0], plain.dumps[0])
    # rows late enough hold more than k of the tied positions among their top scores
    sc = ic.indexer_scores(layers[0]["q_idx"], layers[0]["k_idx"], layers[0]["w"], 0).reshape(-1, 3000)
    t = 2999
    row = sc[t, : t + 1].float()
    top_tie = (row[tied] == row.max()).all().item()
    cut_rows = int(top_tie)
    for t in range(2000, 3000, 97):
        row = sc[t, : t + 1].float()
        vis = tied[tied <= t]
        if (row[vis] == row.max()).all() and vis.numel() > wl.k:
            cut_rows += 1
    assert cut_rows > 0, "no row's top-k cut the tie; the case does not exercise the cut"


def test_fused_8k_prefill_equals_unfused_stack(ic):
    """The benchmarked 8K prefill (8 layers FSSSFSSS, k = 2048), fused and
    unfused: the same index rows in every layer and the same outputs, whose
    rows (all t < 6k = 12288) attend dense-masked over the bitmask the fused selection
    wrote.  Sampled rows also equal the oracle's top-k of the GPU scores."""
    wl = synth.WORKLOADS["prefill_8k"]
    layers = [{n: t.cuda() for n, t in L.items()}
              for L in synth.make_layers(wl, indexer_for_all=False)]
    fused = _stack(ic, wl, layers, 1)
    plain = _stack(ic, wl, layers, 0)
    for l in range(wl.n_layers):
        assert torch.equal(fused.dumps[l], plain.dumps[l]), l
        assert torch.equal(fused.outs[l], plain.outs[l]), l
    rows = synth.sample_rows(wl, 64)
    want = _expected(ic, wl, layers[4], rows)                # the second F layer
    got = fused.dumps[4].cpu().numpy().reshape(-1, wl.k)[rows]
    assert np.array_equal(got, want)


def test_long_rows_fall_back_when_all_scores_tie(ic):
    """w = 0: every score is 0, so every threshold is 0 and every visible
    position is a candidate.  Rows with up to 4k positions fit their lists and
    are selected from their candidates; rows with more than 8k overflow (the
    list holds 4k candidates plus at most 4k reserved-but-unused slots at this
    size) and fall back; rows in between may do either.  Every index row is
    the closed form [0 .. min(k, t+1) - 1] (ties go to the lower position)."""
    wl = synth.Workload("w_zero", 1, 4096, 4096, 2, 32, 128, 256, 16, 128, "FS", 0, 52, True)
    cpu = synth.make_layers(wl)
    cpu[0]["w"] = torch.zeros_like(cpu[0]["w"])
    layers = [{n: t.cuda() for n, t in L.items()} for L in cpu]
    st = _stack(ic, wl, layers, 1)
    QB = 256 // wl.H_I
    fb = st.fused_fallback_blocks()
    assert _blocks_with_long_rows(wl, QB, 8 * wl.k) <= fb <= _blocks_with_long_rows(wl, QB, 4 * wl.k)
    assert fb > 0
    got = st.dumps[0].cpu().numpy().reshape(-1, wl.k)
    t = np.arange(wl.Lq)
    want = np.where(np.arange(wl.k)[None, :] <= t[:, None], np.arange(wl.k)[None, :], -1)
    assert np.array_equal(got, want)
    plain = _stack(ic, wl, layers, 0)
    assert torch.equal(st.outs[0], plain.outs[0]) and torch.equal(st.outs[1], plain.outs[1])


def test_tiny_margin_mixes_fallback_and_fused_rows(ic):
    """z = 0.001 puts the threshold near the sample quantile itself, so about
    half the rows with sampled thresholds (more than 4k positions) find fewer
    than k candidates: their blocks fall back, the others are selected from
    candidates; all rows stay exact."""
    wl = synth.Workload("z_tiny", 1, 6144, 6144, 2, 64, 128, 256, 16, 128, "FS", 0, 53, True)
    layers = [{n: t.cuda() for n, t in L.items()} for L in synth.make_layers(wl)]
    st = _stack(ic, wl, layers, 1, z=0.001)
    QB = 256 // wl.H_I
    fb = st.fused_fallback_blocks()
    assert 0 < fb < _blocks_with_long_rows(wl, QB, 4 * wl.k)
    want = _expected(ic, wl, layers[0])
    assert np.array_equal(st.dumps[0].cpu().numpy().reshape(-1, wl.k), want)


@pytest.mark.parametrize("rows_per_chunk", [256, 1000])
def test_chunked_workspace_with_fallback_rounds(ic, rows_per_chunk):
    """A workspace sized for chunks of a few hundred rows: the rows run in
    several chunks, each with its own thresholds, candidates and 8 fallback
    rounds over a buffer of an eighth of its blocks; a tiny margin makes
    blocks of every chunk fall back."""
    wl = synth.Workload("chunks", 1, 5000, 5000, 2, 32, 128, 128, 16, 128, "FS", 0, 54, True)
    layers = [{n: t.cuda() for n, t in L.items()} for L in synth.make_layers(wl)]
    st = _stack(ic, wl, layers, 1, z=0.001, rows_per_chunk=rows_per_chunk)
    want = _expected(ic, wl, layers[0])
    assert np.array_equal(st.dumps[0].cpu().numpy().reshape(-1, wl.k), want)
    plain = _stack(ic, wl, layers, 0, rows_per_chunk=rows_per_chunk)
    assert torch.equal(st.outs[0], plain.outs[0]) and torch.equal(st.outs[1], plain.outs[1])


def test_indexer_rows_do_not_depend_on_their_query_block(ic):
    """A row's scores are the same bits whichever rows share its query block
    (the full-size tests take expected index rows from row slices of the
    indexer): rows [i0, i0 + n) scored with q_offset = i0 equal those rows
    of the full call."""
    wl = synth.Workload("slices", 1, 2000, 2000, 1, 64, 128, 128, 16, 128, "F", 0, 55, True)
    L = {n: t.cuda() for n, t in synth.make_layers(wl)[0].items()}
    full = ic.indexer_scores(L["q_idx"], L["k_idx"], L["w"], 0)
    for i0, n in ((0, 5), (3, 7), (1001, 999), (1998, 2), (500, 1)):
        part = ic.indexer_scores(L["q_idx"][:, i0:i0 + n].contiguous(), L["k_idx"],
                                 L["w"][:, i0:i0 + n].contiguous(), i0)
        torch.cuda.synchronize()
        assert torch.equal(part[0], full[0, i0:i0 + n])
