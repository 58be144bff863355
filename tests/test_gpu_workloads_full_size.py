"""The layer stack at the full sizes of the benchmarked long-context
configurations, in the configuration bench.py times (inputs drawn on the
device, score chunks as bench.py sizes them):

* prefill: B=1, L=65536, 8 layers FSSSFSSS, indexer 64 x 128, k=2048,
  attention 16 x 128;
* decode: B=32 sequences of one query over 32768 cached positions, 16 layers
  (FSSS)x4;
* the longest single-layer sweep point: L=131072, whose scores take 4
  workspace chunks.

Every row of every layer is checked on the device:

* its index row is valid: min(k, t+1) strictly ascending positions <= t,
  then -1;
* S layers hold exactly their F layer's rows.

A bounded sample of rows is checked against the oracle:

* the index rows of every F layer are bit-exact with the oracle's top-k of
  the GPU's own indexer scores of those rows (at 64K and 128K the stack
  fuses the top-k into the indexer and never stores the score matrix; the
  rows' scores come from ic_indexer_scores on the rows alone);
* top-k set overlap >= 0.99 against the oracle's own scores;
* attention within the tolerance against the oracle's attention over the
  GPU's own index rows.  At 64K a row rarely has exactly the oracle's set,
  so every sampled row is compared this way.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from lightning_indexer_top_relu_b200 import build, synth

pytestmark = pytest.mark.gpu

ATTN_ATOL = 2e-2
LSE_ATOL = 1e-3


@pytest.fixture(scope="module")
def ic():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    from lightning_indexer_top_relu_b200 import indexcache
    return indexcache


def _valid_rows(idx: torch.Tensor, q_offset: int, k: int) -> bool:
    B, Lq, _ = idx.shape
    t = torch.arange(Lq, device=idx.device) + q_offset
    m = torch.clamp(t + 1, max=k)
    slot = torch.arange(k, device=idx.device)
    valid = slot[None, :] < m[:, None]
    ok = torch.all(torch.where(valid[None], (idx >= 0) & (idx <= t[None, :, None]), idx == -1))
    d = idx[..., 1:] - idx[..., :-1]
    return bool(ok) and bool(torch.all(torch.where(valid[None, :, 1:], d > 0, True)))


def bench_rows_per_chunk(wl) -> int:
    """F-layer score rows per workspace chunk as bench.py sizes them: as many
    as 16 GiB of fp32 scores hold."""
    return max(1, min(wl.B * wl.Lq, (16 * 2 ** 30) // (4 * wl.Lk)))


def topk_of_gpu_rows(ic, wl, L, rows):
    """The oracle's top-k of the GPU indexer's scores of flattened rows
    `rows`, each scored alone (a one-row call at its own position; a row's
    scores do not depend on the rows sharing its query block)."""
    out = []
    for r in rows:
        b, i = divmod(int(r), wl.Lq)
        sc = ic.indexer_scores(L["q_idx"][b:b + 1, i:i + 1].contiguous(), L["k_idx"][b:b + 1],
                               L["w"][b:b + 1, i:i + 1].contiguous(), wl.q_offset + i)
        out.append(sc.reshape(1, wl.Lk).cpu().numpy())
    tpos = oracle.row_positions(wl.B, wl.Lq, wl.q_offset, rows)
    return oracle.topk_sort(np.concatenate(out), tpos, wl.k)


def check_sampled(ic, wl, layers, ref_layers, ref_wl, rows, ref_rows, sync):
    """Runs the stack on `layers` (device tensors) and checks it as the
    module docstring says.  The oracle runs on `ref_layers` (CPU tensors of
    the problem `ref_wl`, the same sequences or a sub-batch of them): its
    flattened row ref_rows[j] is the stack's row rows[j]."""
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    st = ic.LayerStack(wl.pattern, layers, dims, want_lse=True, dump_idx=True,
                       rows_per_chunk=bench_rows_per_chunk(wl))
    st.forward()
    sync()
    assert ic.get_last_device_error() == 0
    src = 0
    for l, c in enumerate(wl.pattern):
        if c in "F1":
            src = l
        assert _valid_rows(st.dumps[l], wl.q_offset, wl.k), l
        assert torch.equal(st.dumps[l], st.dumps[src]), l
    _, ref_idx, _ = oracle.layer_stack(ref_wl.pattern, ref_layers, ref_wl.k, ref_wl.q_offset,
                                       rows=ref_rows)
    sel = torch.as_tensor(np.asarray(rows, dtype=np.int64), device=st.dumps[0].device)
    for l, c in enumerate(wl.pattern):
        if c in "F1":
            want = topk_of_gpu_rows(ic, wl, layers[l], rows)
            assert np.array_equal(st.dumps[l].reshape(-1, wl.k)[sel].cpu().numpy(), want), l
    for l in range(wl.n_layers):
        gidx = st.dumps[l].reshape(-1, wl.k)[sel].cpu().numpy()
        ov = [len(set(a[a >= 0].tolist()) & set(b[b >= 0].tolist())) / max(int((b >= 0).sum()), 1)
              for a, b in zip(gidx, ref_idx[l])]
        assert np.mean(ov) >= 0.99, (l, np.mean(ov), min(ov))
        L = ref_layers[l]
        ref, ref_lse = oracle.sparse_attn(L["q"], L["k"], L["v"], gidx, ref_wl.q_offset,
                                          rows=ref_rows)
        out = st.outs[l].reshape(-1, wl.Hq, wl.d)[sel].float().cpu().numpy()
        lse = st.lses[l].reshape(-1, wl.Hq)[sel].cpu().numpy()
        assert np.abs(out - ref).max() <= ATTN_ATOL, l
        assert np.abs(lse - ref_lse).max() <= LSE_ATOL, l


def test_prefill_64k_stack_full_size_sampled_rows(ic):
    wl = synth.WORKLOADS["prefill_64k"]
    layers = synth.make_layers(wl, indexer_for_all=False, device="cuda")   # drawn as bench.py does
    ref_layers = [{n: t.cpu() for n, t in L.items()} for L in layers]
    rows = synth.sample_rows(wl, 24)
    check_sampled(ic, wl, layers, ref_layers, wl, rows, rows, torch.cuda.synchronize)


def test_decode_32k_stack_full_size_sampled_rows(ic):
    wl = synth.WORKLOADS["decode_32k"]
    layers = synth.make_layers(wl, indexer_for_all=False, device="cuda")
    seqs = list(range(0, wl.B, 4))                        # the oracle sees 8 of the 32 sequences
    ref_layers = [{n: t[seqs].cpu() for n, t in L.items()} for L in layers]
    ref_wl = dataclasses.replace(wl, B=len(seqs))
    check_sampled(ic, wl, layers, ref_layers, ref_wl, seqs, list(range(len(seqs))),
                  torch.cuda.synchronize)


def test_sweep_128k_layer_full_size_chunked_scores(ic):
    """One F layer at L = 131072 with the workspace bench.py gives it (16 GiB
    of scores: 4 chunks of 32768 rows on the plain path; the fused top-k,
    which the stack takes here, fits its candidate lists in fewer)."""
    wl = synth.WORKLOADS["sweep_128k"]
    assert bench_rows_per_chunk(wl) == 32768
    layers = synth.make_layers(wl, device="cuda")
    ref_layers = [{n: t.cpu() for n, t in L.items()} for L in layers]
    rows = synth.sample_rows(wl, 24)
    check_sampled(ic, wl, layers, ref_layers, wl, rows, rows, torch.cuda.synchronize)


def _score_rel_err(gpu: np.ndarray, ref: np.ndarray, tpos) -> float:
    """Largest |gpu - ref| / max(|ref|, 1e-3 * max |ref row|) over visible
    positions (the floor keeps sign-mixed rows from dividing by ~0)."""
    worst = 0.0
    for r, t in enumerate(tpos):
        g, f = gpu[r, : t + 1].astype(np.float64), ref[r, : t + 1]
        floor = 1e-3 * max(np.abs(f).max(), 1e-30)
        worst = max(worst, float((np.abs(g - f) / np.maximum(np.abs(f), floor)).max()))
    return worst


def check_kernels_one_by_one(ic, wl, L, sync):
    """Each step on its own over a whole layer (`L`, device tensors): indexer
    scores within 2e-2 of the oracle's (invisible positions exactly -inf),
    top-k bit-exact on the GPU's own scores, gather attention within the
    attention tolerance on the GPU's own index rows -- on sampled rows."""
    rows = synth.sample_rows(wl, 24)
    dev = L["q"].device
    sel = torch.as_tensor(np.asarray(rows, dtype=np.int64), device=dev)
    tpos = oracle.row_positions(wl.B, wl.Lq, wl.q_offset, rows)
    cpu = {n: t.cpu() for n, t in L.items()}

    scores = ic.indexer_scores(L["q_idx"], L["k_idx"], L["w"], wl.q_offset)
    sync()
    got = scores.reshape(-1, wl.Lk)[sel].cpu().numpy()
    ref = oracle.indexer_scores(cpu["q_idx"], cpu["k_idx"], cpu["w"], wl.q_offset, rows=rows)
    assert _score_rel_err(got, ref, tpos) <= 2e-2
    for r, t in enumerate(tpos):
        assert np.all(np.isneginf(got[r, t + 1:]))

    idx = ic.topk_select(scores, wl.k, wl.q_offset)
    del scores
    gidx = idx.reshape(-1, wl.k)[sel].cpu().numpy()
    assert np.array_equal(gidx, oracle.topk_sort(got, tpos, wl.k))

    out, lse = ic.sparse_attn(L["q"], L["k"], L["v"], idx, wl.q_offset)
    assert ic.get_last_device_error() == 0
    ref_o, ref_lse = oracle.sparse_attn(cpu["q"], cpu["k"], cpu["v"], gidx, wl.q_offset, rows=rows)
    assert np.abs(out.reshape(-1, wl.Hq, wl.d)[sel].float().cpu().numpy() - ref_o).max() <= ATTN_ATOL
    assert np.abs(lse.reshape(-1, wl.Hq)[sel].cpu().numpy() - ref_lse).max() <= LSE_ATOL


@pytest.mark.parametrize("name", ["prefill_8k", "prefill_64k"])
def test_kernels_one_by_one_full_size_sampled_rows(ic, name):
    wl = synth.WORKLOADS[name]
    L = synth.make_layers(wl, layers=[0], device="cuda")[0]
    check_kernels_one_by_one(ic, wl, L, torch.cuda.synchronize)
