"""ic_sparse_attn_no_alloc against ic_sparse_attn, through the C ABI.

The no-allocation entry point serves callers that cannot give the library any
device memory of its own (a host framework that owns every GPU buffer and
passes a plugin only its inputs and outputs; a decode loop that must not call
cudaMalloc).  Its results must match the workspace-based entry point within
the attention tolerance, on two calls in a row: the second call runs on other
inputs and must not see anything the first call left in the shared scratch.

This file is named to be collected last, so a run that stops at the first
failure has run every other test before it.  It passes both alone in a fresh
process and after the rest of the suite.
"""
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


def _decode_case(cfg_id):
    # decode rows: few rows, so the slots of each row are split over several
    # CTAs and the per-split partials go through the scratch
    wl = synth.custom(B=4, Lq=1, Lk=3000, q_offset=2999, H_I=4, d_I=64, k=2048, Hq=16, d=128,
                      cfg_id=cfg_id)
    L = synth.make_layers(wl)[0]
    sc = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"], wl.q_offset).astype(np.float32)
    idx = oracle.topk_sort(sc, oracle.row_positions(wl.B, 1, wl.q_offset), wl.k)
    dev = {n: L[n].cuda() for n in ("q", "k", "v")}
    return wl, dev, torch.from_numpy(idx).reshape(wl.B, 1, wl.k).cuda()


def test_no_alloc_matches_workspace_entry_point_twice(ic):
    assert ic.sparse_attn_workspace_bytes(4, 1, 16, 128, 2048) > 0    # the split path is taken
    for cfg_id in (31, 32):                                           # two calls in a row
        wl, t, idx = _decode_case(cfg_id)
        ref, ref_lse = ic.sparse_attn(t["q"], t["k"], t["v"], idx, wl.q_offset)
        out, lse = ic.sparse_attn_no_alloc(t["q"], t["k"], t["v"], idx, wl.q_offset)
        torch.cuda.synchronize()
        assert ic.get_last_device_error() == 0
        assert (out.float() - ref.float()).abs().max().item() <= ATTN_ATOL
        assert (lse - ref_lse).abs().max().item() <= LSE_ATOL


@pytest.mark.parametrize("B", [100, 300])
def test_no_alloc_runs_calls_of_many_rows(ic, B):
    # 100 rows still split their slots, over a thread-block cluster per row
    # that merges in distributed shared memory (the scratch stays unused; the
    # workspace query still counts the partials a cluster-less device would
    # need); 300 rows fill the CTAs the GPU holds at once and run one split
    # each.  Both equal the workspace entry point.
    wl = synth.custom(B=B, Lq=1, Lk=600, q_offset=599, H_I=4, d_I=64, k=256, Hq=16, d=128,
                      cfg_id=33)
    assert (ic.sparse_attn_workspace_bytes(B, 1, 16, 128, 256) > 0) == (B == 100)
    L = synth.make_layers(wl)[0]
    sc = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"], wl.q_offset).astype(np.float32)
    idx = oracle.topk_sort(sc, oracle.row_positions(wl.B, 1, wl.q_offset), wl.k)
    t = {n: L[n].cuda() for n in ("q", "k", "v")}
    idx_d = torch.from_numpy(idx).reshape(wl.B, 1, wl.k).cuda()
    ref, ref_lse = ic.sparse_attn(t["q"], t["k"], t["v"], idx_d, wl.q_offset)
    out, lse = ic.sparse_attn_no_alloc(t["q"], t["k"], t["v"], idx_d, wl.q_offset)
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    assert (out.float() - ref.float()).abs().max().item() <= ATTN_ATOL
    assert (lse - ref_lse).abs().max().item() <= LSE_ATOL
