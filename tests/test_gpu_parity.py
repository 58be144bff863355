"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Bars (stated for bf16 inputs with fp32 accumulation):
  * indexer scores: max relative error <= 2e-2, where the error of a score is
    |gpu - oracle| / max(|oracle|, 1e-3 * max |oracle row|) (the floor keeps
    sign-mixed rows from dividing by ~0); masked positions exactly -inf;
  * top-k on the same fp32 score tensor (drawn on the CPU or computed by the
    oracle): bit-exact;
  * sparse attention on the same index tensor: max abs error <= 2e-2 on the
    bf16 output, <= 1e-3 on the log-sum-exp;
  * layer stack end to end: mean top-k set overlap >= 0.99 against the
    oracle's own scores, attention outputs within 2e-2 on the rows whose
    sets agree, S-layer indices bitwise equal to their F layer's.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from lightning_indexer_top_relu_b200 import build, synth

pytestmark = pytest.mark.gpu

SCORE_RTOL = 2e-2
ATTN_ATOL = 2e-2
LSE_ATOL = 1e-3


@pytest.fixture(scope="module")
def ic():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    from lightning_indexer_top_relu_b200 import indexcache
    return indexcache


def _cuda(layer):
    return {k: v.cuda() for k, v in layer.items()}


def score_rel_err(gpu: np.ndarray, ref: np.ndarray, tpos) -> float:
    worst = 0.0
    for r, t in enumerate(tpos):
        g, f = gpu[r, : t + 1].astype(np.float64), ref[r, : t + 1]
        floor = 1e-3 * max(np.abs(f).max(), 1e-30)
        worst = max(worst, float((np.abs(g - f) / np.maximum(np.abs(f), floor)).max()))
    return worst


def overlap(a: np.ndarray, b: np.ndarray):
    out = []
    for ra, rb in zip(a.reshape(-1, a.shape[-1]), b.reshape(-1, b.shape[-1])):
        sa, sb = set(ra[ra >= 0].tolist()), set(rb[rb >= 0].tolist())
        out.append(len(sa & sb) / max(len(sa), 1))
    return np.array(out)


def check_idx_valid(idx: torch.Tensor, q_offset: int, k: int):
    """Every row: min(k, t+1) strictly ascending positions in [0, t], then -1."""
    B, Lq, _ = idx.shape
    t = torch.arange(Lq, device=idx.device) + q_offset
    m = torch.clamp(t + 1, max=k)
    slot = torch.arange(k, device=idx.device)
    valid = slot[None, :] < m[:, None]
    assert torch.all(torch.where(valid[None], idx >= 0, idx == -1))
    assert torch.all(torch.where(valid[None], idx <= t[None, :, None], True))
    d = idx[..., 1:] - idx[..., :-1]
    assert torch.all(torch.where(valid[None, :, 1:], d > 0, True))


# ------------------------------------------------------------------ indexer

INDEXER_SHAPES = [
    # B, Lq, Lk, q_offset, H_I, d_I
    (1, 512, 512, 0, 4, 64),       # the tiny prefill layer shape
    (2, 1000, 1000, 0, 32, 128),   # ragged tail, several key tiles, B > 1
    (1, 129, 129, 0, 64, 128),
    (1, 1, 1, 0, 8, 64),
    (3, 1, 700, 699, 64, 128),     # decode rows
    (2, 100, 300, 200, 16, 64),    # rows in the middle of a sequence
    (1, 300, 300, 0, 128, 64),
]


@pytest.mark.parametrize("B,Lq,Lk,q_offset,H,dI", INDEXER_SHAPES)
def test_indexer_scores_match_oracle(ic, B, Lq, Lk, q_offset, H, dI):
    wl = synth.custom(B=B, Lq=Lq, Lk=Lk, q_offset=q_offset, H_I=H, d_I=dI, k=8, cfg_id=21)
    L = synth.make_layers(wl)[0]
    ref = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"], q_offset)
    gpu = ic.indexer_scores(L["q_idx"].cuda(), L["k_idx"].cuda(), L["w"].cuda(), q_offset)
    gpu = gpu.cpu().numpy().reshape(B * Lq, Lk)
    tpos = oracle.row_positions(B, Lq, q_offset)
    assert score_rel_err(gpu, ref, tpos) <= SCORE_RTOL
    mask = np.isneginf(ref)
    assert np.array_equal(np.isneginf(gpu), mask)


def test_indexer_small_integers_are_bit_exact(ic):
    """Small-integer bf16 operands and dyadic w: every product and partial sum
    is exact in fp32, so the tensor-core path must equal the oracle exactly."""
    rng = np.random.default_rng(11)
    B, L, H, dI = 1, 300, 4, 64
    q = torch.tensor(rng.integers(-3, 4, (B, L, H, dI)), dtype=torch.bfloat16)
    k = torch.tensor(rng.integers(-3, 4, (B, L, dI)), dtype=torch.bfloat16)
    w = torch.tensor(rng.choice([-2.0, -1.0, 0.5, 1.0, 2.0], (B, L, H)), dtype=torch.float32)
    ref = oracle.indexer_scores(q, k, w).astype(np.float32)
    gpu = ic.indexer_scores(q.cuda(), k.cuda(), w.cuda()).cpu().numpy().reshape(L, L)
    assert np.array_equal(gpu, ref)


# ------------------------------------------------------------------ top-k

def _score_draw(kind, rows, Lk, seed):
    rng = np.random.default_rng(seed)
    if kind == "gauss":
        return rng.normal(size=(rows, Lk)).astype(np.float32)
    if kind == "ties":
        return rng.integers(-2, 3, size=(rows, Lk)).astype(np.float32)
    if kind == "zeros":
        s = np.where(rng.random((rows, Lk)) < 0.5, np.float32(-0.0), np.float32(0.0))
        s[:, ::5] = rng.normal(size=s[:, ::5].shape).astype(np.float32)
        return s
    if kind == "const":
        return np.full((rows, Lk), 0.25, dtype=np.float32)
    if kind == "tiny":
        return (rng.normal(size=(rows, Lk)) * 1e-30).astype(np.float32)
    raise ValueError(kind)


TOPK_CASES = [
    # B, Lq, Lk, q_offset, k, draw
    (1, 512, 512, 0, 64, "gauss"),
    (2, 1000, 1000, 0, 100, "ties"),
    (1, 700, 700, 0, 1, "gauss"),
    (1, 300, 300, 0, 300, "gauss"),        # k = L: every row keeps everything
    (1, 600, 600, 0, 37, "zeros"),         # signed zeros must tie
    (1, 400, 400, 0, 50, "const"),         # all ties -> lowest positions
    (1, 400, 400, 0, 50, "tiny"),          # denormal-range values
    (1, 5000, 5000, 0, 2048, "gauss"),     # the stack's k over multi-tile rows
    (4, 1, 9000, 8999, 2048, "gauss"),     # decode rows
    (1, 6, 50000, 49994, 2048, "gauss"),   # rows too long for shared memory
]


@pytest.mark.parametrize("B,Lq,Lk,q_offset,k,draw", TOPK_CASES)
def test_topk_bit_exact_on_shared_scores(ic, B, Lq, Lk, q_offset, k, draw):
    sc = _score_draw(draw, B * Lq, Lk, seed=Lk + k)
    tpos = oracle.row_positions(B, Lq, q_offset)
    ref = oracle.topk_sort(sc, tpos, k)
    gpu = ic.topk_select(torch.from_numpy(sc).reshape(B, Lq, Lk).cuda(), k, q_offset)
    assert np.array_equal(gpu.cpu().numpy().reshape(B * Lq, k), ref)


def test_topk_on_oracle_indexer_scores(ic):
    wl = synth.WORKLOADS["tiny_prefill"]
    L = synth.make_layers(wl, layers=[0])[0]
    sc = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"]).astype(np.float32)
    ref = oracle.topk_sort(sc, oracle.row_positions(1, 512, 0), wl.k)
    gpu = ic.topk_select(torch.from_numpy(sc).reshape(1, 512, 512).cuda(), wl.k)
    assert np.array_equal(gpu.cpu().numpy().reshape(512, wl.k), ref)


# ------------------------------------------------------------------ sparse attention

def _oracle_idx(L, k, q_offset):
    B, Lq = L["q_idx"].shape[:2]
    sc = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"], q_offset).astype(np.float32)
    return oracle.topk_sort(sc, oracle.row_positions(B, Lq, q_offset), k)


ATTN_CASES = [
    # B, Lq, Lk, q_offset, Hq, d, k
    (1, 512, 512, 0, 8, 64, 64),
    (2, 300, 300, 0, 16, 128, 100),
    (4, 1, 3000, 2999, 16, 128, 2048),     # decode: 32 splits, workspace + combine kernel
    (40, 1, 3000, 2999, 16, 128, 2048),    # decode: 7 splits, one 7-CTA cluster per row
    (20, 1, 3000, 2999, 16, 128, 2048),    # decode: 14 splits trimmed to one 8-CTA cluster
    (37, 1, 5000, 4999, 16, 64, 1024),     # decode, d = 64: 8 splits in a cluster
    (1, 200, 200, 0, 16, 64, 256),         # k > L: padded tails
]


@pytest.mark.parametrize("B,Lq,Lk,q_offset,Hq,d,k", ATTN_CASES)
def test_sparse_attn_matches_oracle(ic, B, Lq, Lk, q_offset, Hq, d, k):
    wl = synth.custom(B=B, Lq=Lq, Lk=Lk, q_offset=q_offset, H_I=4, d_I=64, k=k, Hq=Hq, d=d,
                      cfg_id=22)
    L = synth.make_layers(wl)[0]
    idx = _oracle_idx(L, k, q_offset)
    ref, ref_lse = oracle.sparse_attn(L["q"], L["k"], L["v"], idx, q_offset)
    out, lse = ic.sparse_attn(L["q"].cuda(), L["k"].cuda(), L["v"].cuda(),
                              torch.from_numpy(idx).reshape(B, Lq, k).cuda(), q_offset)
    assert ic.get_last_device_error() == 0
    got = out.float().cpu().numpy().reshape(B * Lq, Hq, d)
    assert np.abs(got - ref).max() <= ATTN_ATOL
    assert np.abs(lse.cpu().numpy().reshape(B * Lq, Hq) - ref_lse).max() <= LSE_ATOL


def test_clustered_decode_splits_without_valid_slots(ic):
    """Decode rows whose valid slots all sit in the first split: the other
    splits of the row's cluster hold no slot (log-sum-exp -inf) and the
    merge through distributed shared memory must weigh them 0; one row has
    no valid slot at all (out 0, lse -inf)."""
    B, Lk, Hq, d, k = 40, 3000, 16, 128, 2048
    wl = synth.custom(B=B, Lq=1, Lk=Lk, q_offset=Lk - 1, H_I=4, d_I=64, k=k, Hq=Hq, d=d, cfg_id=24)
    lay = synth.make_layers(wl)[0]
    rng = np.random.default_rng(5)
    idx = np.full((B, k), -1, dtype=np.int32)
    for b in range(1, B):
        n = int(rng.integers(1, 200))
        idx[b, :n] = rng.choice(Lk, size=n, replace=False)
    ref, ref_lse = oracle.sparse_attn(lay["q"], lay["k"], lay["v"], idx, Lk - 1)
    out, lse = ic.sparse_attn(lay["q"].cuda(), lay["k"].cuda(), lay["v"].cuda(),
                              torch.from_numpy(idx).reshape(B, 1, k).cuda(), Lk - 1)
    assert ic.get_last_device_error() == 0
    got = out.float().cpu().numpy().reshape(B, Hq, d)
    assert np.abs(got - ref).max() <= ATTN_ATOL
    assert np.all(got[0] == 0.0)
    g_lse = lse.cpu().numpy().reshape(B, Hq)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(g_lse), fin) and not fin[0].any()
    assert np.abs(g_lse[fin] - ref_lse[fin]).max() <= LSE_ATOL


def test_sparse_attn_with_holes_and_bad_indices(ic):
    """-1 slots anywhere are empty; an index beyond t is skipped and reported
    through the device error word (no fault)."""
    B, L, Hq, d, k = 1, 160, 16, 128, 40
    wl = synth.custom(B=B, Lq=L, H_I=4, d_I=64, k=k, Hq=Hq, d=d, cfg_id=23)
    lay = synth.make_layers(wl)[0]
    rng = np.random.default_rng(3)
    idx = np.full((L, k), -1, dtype=np.int32)
    for t in range(L):
        cand = rng.choice(t + 1, size=min(k, t + 1), replace=False)
        keep = rng.random(len(cand)) < 0.7
        idx[t, : len(cand)] = np.where(keep, cand, -1)
    rng.shuffle(idx, axis=1)
    ref, ref_lse = oracle.sparse_attn(lay["q"], lay["k"], lay["v"], idx)
    out, lse = ic.sparse_attn(lay["q"].cuda(), lay["k"].cuda(), lay["v"].cuda(),
                              torch.from_numpy(idx).reshape(1, L, k).cuda())
    assert ic.get_last_device_error() == 0
    got = out.float().cpu().numpy().reshape(L, Hq, d)
    assert np.abs(got - ref).max() <= ATTN_ATOL
    fin = np.isfinite(ref_lse)
    g_lse = lse.cpu().numpy().reshape(L, Hq)
    assert np.array_equal(np.isfinite(g_lse), fin)
    assert np.abs(g_lse[fin] - ref_lse[fin]).max() <= LSE_ATOL

    bad = idx.copy()
    bad[100, 0] = 150            # beyond t = 100
    out2, _ = ic.sparse_attn(lay["q"].cuda(), lay["k"].cuda(), lay["v"].cuda(),
                             torch.from_numpy(bad).reshape(1, L, k).cuda())
    assert ic.get_last_device_error() == 1          # IC_ERR_INVALID_ARG, context still usable
    bad_ref = bad.copy()
    bad_ref[100, 0] = -1
    ref2, _ = oracle.sparse_attn(lay["q"], lay["k"], lay["v"], bad_ref)
    assert np.abs(out2.float().cpu().numpy().reshape(L, Hq, d) - ref2).max() <= ATTN_ATOL
    assert ic.get_last_device_error() == 0


DENSE_CASES = [
    # B, Lq, Lk, q_offset, Hq, d, k   (rows t < 6k take the dense-masked kernel)
    (1, 700, 700, 0, 16, 128, 48),          # 36 dense blocks, 412 gathered rows
    (1, 700, 700, 0, 16, 128, 96),          # 72 dense blocks, 124 gathered rows split over CTAs
    (2, 1000, 1000, 0, 16, 128, 256),       # all dense, B = 2, ragged last key tile
    (1, 300, 1324, 1024, 16, 128, 512),     # mid-sequence chunk, 4 gathered tail rows (8 splits)
    (1, 500, 500, 0, 8, 128, 128),          # 16 queries per block
]


@pytest.mark.parametrize("B,Lq,Lk,q_offset,Hq,d,k", DENSE_CASES)
def test_unique_attn_dense_and_gathered_rows_match_oracle(ic, B, Lq, Lk, q_offset, Hq, d, k):
    wl = synth.custom(B=B, Lq=Lq, Lk=Lk, q_offset=q_offset, H_I=4, d_I=64, k=k, Hq=Hq, d=d,
                      cfg_id=27)
    L = synth.make_layers(wl)[0]
    idx = _oracle_idx(L, k, q_offset)
    ref, ref_lse = oracle.sparse_attn(L["q"], L["k"], L["v"], idx, q_offset)
    t = {n: L[n].cuda() for n in ("q", "k", "v")}
    idx_d = torch.from_numpy(idx).reshape(B, Lq, k).cuda()
    n0 = ic.kernel_launch_count()
    out, lse = ic.sparse_attn_unique(t["q"], t["k"], t["v"], idx_d, q_offset)
    n_dense = ic.kernel_launch_count() - n0
    assert ic.get_last_device_error() == 0
    assert n_dense >= 3                                  # mask build, V^T, dense kernel
    got = out.float().cpu().numpy().reshape(B * Lq, Hq, d)
    assert np.abs(got - ref).max() <= ATTN_ATOL
    assert np.abs(lse.cpu().numpy().reshape(B * Lq, Hq) - ref_lse).max() <= LSE_ATOL
    # without the workspace every row gathers: the same results
    out_g, lse_g = ic.sparse_attn_unique(t["q"], t["k"], t["v"], idx_d, q_offset,
                                         ws=torch.empty(0, device="cuda", dtype=torch.uint8))
    assert ic.get_last_device_error() == 0
    assert (out_g.float() - out.float()).abs().max().item() <= ATTN_ATOL
    assert (lse_g - lse).abs().max().item() <= LSE_ATOL


def test_unique_attn_dense_rows_with_holes_and_bad_indices(ic):
    """The dense-masked kernel sees the selection only as a bitmask: -1 slots
    anywhere, unsorted rows, and an index beyond t (skipped and reported)."""
    B, L, Hq, d, k = 1, 160, 16, 128, 40                 # every row t < 6k = 240
    wl = synth.custom(B=B, Lq=L, H_I=4, d_I=64, k=k, Hq=Hq, d=d, cfg_id=28)
    lay = synth.make_layers(wl)[0]
    rng = np.random.default_rng(5)
    idx = np.full((L, k), -1, dtype=np.int32)
    for t in range(L):
        cand = rng.choice(t + 1, size=min(k, t + 1), replace=False)
        keep = rng.random(len(cand)) < 0.7
        idx[t, : len(cand)] = np.where(keep, cand, -1)
    rng.shuffle(idx, axis=1)
    ref, ref_lse = oracle.sparse_attn(lay["q"], lay["k"], lay["v"], idx)
    q, kk, v = lay["q"].cuda(), lay["k"].cuda(), lay["v"].cuda()
    out, lse = ic.sparse_attn_unique(q, kk, v, torch.from_numpy(idx).reshape(1, L, k).cuda())
    assert ic.get_last_device_error() == 0
    assert np.abs(out.float().cpu().numpy().reshape(L, Hq, d) - ref).max() <= ATTN_ATOL
    fin = np.isfinite(ref_lse)
    g_lse = lse.cpu().numpy().reshape(L, Hq)
    assert np.array_equal(np.isfinite(g_lse), fin)
    assert np.abs(g_lse[fin] - ref_lse[fin]).max() <= LSE_ATOL

    bad = idx.copy()
    slot = int(np.flatnonzero(bad[100] == -1)[0])
    bad[100, slot] = 150                                  # beyond t = 100
    out2, _ = ic.sparse_attn_unique(q, kk, v, torch.from_numpy(bad).reshape(1, L, k).cuda())
    assert ic.get_last_device_error() == 1                # IC_ERR_INVALID_ARG, context usable
    assert np.abs(out2.float().cpu().numpy().reshape(L, Hq, d) - ref).max() <= ATTN_ATOL
    assert ic.get_last_device_error() == 0


def _first_tile_empty_idx(L, k, seed):
    """Index rows where even queries past position 64 select nothing among
    keys 0..63 and odd queries select key 0: within one warp (two queries x
    16 heads) some rows raise their running max at the second key tile and
    others do not."""
    rng = np.random.default_rng(seed)
    idx = np.full((L, k), -1, dtype=np.int32)
    for t in range(L):
        lo = 64 if (t % 2 == 0 and t >= 64 + k) else 0
        pick = rng.choice(np.arange(lo, t + 1), size=min(k, t + 1 - lo), replace=False)
        if lo == 0 and 0 not in pick:
            pick[0] = 0
        idx[t, : len(pick)] = np.sort(pick)
    return idx


def test_unique_attn_rows_raising_their_max_after_the_first_tile(ic):
    """Rows of one warp raise the running max at different tiles; the O
    rescale in TMEM is warp-collective and must stay correct for all rows."""
    B, L, Hq, d, k = 1, 256, 16, 128, 40                  # rows t < 6k = 240 dense, 16 gather
    wl = synth.custom(B=B, Lq=L, H_I=4, d_I=64, k=k, Hq=Hq, d=d, cfg_id=30)
    lay = synth.make_layers(wl)[0]
    idx = _first_tile_empty_idx(L, k, 11)
    ref, ref_lse = oracle.sparse_attn(lay["q"], lay["k"], lay["v"], idx)
    out, lse = ic.sparse_attn_unique(lay["q"].cuda(), lay["k"].cuda(), lay["v"].cuda(),
                                     torch.from_numpy(idx).reshape(1, L, k).cuda())
    assert ic.get_last_device_error() == 0
    assert np.abs(out.float().cpu().numpy().reshape(L, Hq, d) - ref).max() <= ATTN_ATOL
    assert np.abs(lse.cpu().numpy().reshape(L, Hq) - ref_lse).max() <= LSE_ATOL


# ------------------------------------------------------------------ index cache and layer stack

def _run_stack(ic, wl, layers, pattern=None, **kw):
    pattern = pattern or wl.pattern
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    st = ic.LayerStack(pattern, [_cuda(L) for L in layers], dims, want_lse=True, dump_idx=True,
                       **kw)
    st.forward()
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    return st


def _compare_stack(st, wl, layers, rows, pattern=None):
    pattern = pattern or wl.pattern
    outs, idxs, _ = oracle.layer_stack(pattern, layers, wl.k, wl.q_offset, rows=rows)
    rows_a = np.arange(wl.B * wl.Lq) if rows is None else np.asarray(rows)
    src = 0
    for l, c in enumerate(pattern):
        if c in "F1":
            src = l
        gidx = st.dumps[l].cpu().numpy().reshape(-1, wl.k)
        assert np.array_equal(gidx, st.dumps[src].cpu().numpy().reshape(-1, wl.k))
        g = gidx[rows_a]
        ov = overlap(g, idxs[l])
        assert ov.mean() >= 0.99, (l, ov.mean(), ov.min())
        same = np.array([np.array_equal(a, b) for a, b in zip(g, idxs[l])])
        got = st.outs[l].float().cpu().numpy().reshape(-1, wl.Hq, wl.d)[rows_a]
        assert np.abs(got[same] - outs[l][same]).max() <= ATTN_ATOL
    return True


def test_stack_tiny_prefill_matches_oracle(ic):
    wl = synth.WORKLOADS["tiny_prefill"]
    layers = synth.make_layers(wl)
    st = _run_stack(ic, wl, layers)
    check_idx_valid(st.idx_cache, 0, wl.k)
    _compare_stack(st, wl, layers, None)


def test_stack_chunking_and_pattern_spelling_do_not_change_results(ic):
    wl = synth.custom(Lq=700, n_layers=4, H_I=32, d_I=128, k=96, Hq=16, d=128,
                      pattern="FSFS", cfg_id=24)
    layers = synth.make_layers(wl)
    n0 = ic.kernel_launch_count()
    a = _run_stack(ic, wl, layers)
    assert ic.kernel_launch_count() > n0
    b = _run_stack(ic, wl, layers, pattern="1010", rows_per_chunk=1)   # one query block per chunk
    for l in range(4):
        assert torch.equal(a.outs[l], b.outs[l])
        assert torch.equal(a.dumps[l], b.dumps[l])
    _compare_stack(a, wl, layers, None)


def test_stack_batch_of_two_with_dense_rows(ic):
    # B = 2: the top-k writes each sequence's bitmask rows (b * rows + i) and
    # the dense-masked kernel reads them back
    wl = synth.custom(B=2, Lq=300, n_layers=2, H_I=32, d_I=128, k=64, Hq=16, d=128, pattern="FS",
                      cfg_id=34)
    layers = synth.make_layers(wl)
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    assert ic.layer_stack_dense_rows(dims, ic.layer_stack_workspace_bytes(dims, 2)) == 296
    st = _run_stack(ic, wl, layers)
    check_idx_valid(st.idx_cache, 0, wl.k)
    _compare_stack(st, wl, layers, None)


def test_stack_continuation_chunk_with_dense_rows(ic):
    # rows 512..767 of a sequence whose first 512 positions are already cached
    wl = synth.custom(Lq=256, Lk=768, q_offset=512, n_layers=2, H_I=32, d_I=128, k=128, Hq=16,
                      d=128, pattern="FS", cfg_id=35)
    layers = synth.make_layers(wl)
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    assert ic.layer_stack_dense_rows(dims, ic.layer_stack_workspace_bytes(dims, 2)) == 256
    st = _run_stack(ic, wl, layers)
    check_idx_valid(st.idx_cache, wl.q_offset, wl.k)
    _compare_stack(st, wl, layers, None)


def test_stack_timing_marks_are_recorded_in_order(ic):
    # rows t < 6k take the dense-masked kernel, the rest gather: every mark
    # of every layer is recorded, in stream order
    wl = synth.custom(Lq=700, n_layers=2, H_I=32, d_I=128, k=96, Hq=16, d=128, pattern="FS",
                      cfg_id=26)
    layers = synth.make_layers(wl)
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    st = ic.LayerStack(wl.pattern, [_cuda(L) for L in layers], dims)
    stream = torch.cuda.current_stream()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(ic.MARKS_PER_LAYER * 2)]
    for e in evs:
        e.record(stream)
    arr = (ctypes.c_void_p * len(evs))(*[e.cuda_event for e in evs])
    torch.cuda.synchronize()
    st.forward(stream, events=arr)
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    gaps = [evs[i].elapsed_time(evs[i + 1]) for i in range(len(evs) - 1)]
    assert min(gaps) >= 0.0
    npl = ic.MARKS_PER_LAYER
    assert evs[2].elapsed_time(evs[3]) > 0.0          # layer 0: dense-masked rows
    assert evs[3].elapsed_time(evs[4]) > 0.0          # layer 0: gathered rows
    assert evs[npl + 3].elapsed_time(evs[npl + 4]) > 0.0


def test_stack_leading_shared_layer_fails_before_launch(ic):
    wl = synth.custom(Lq=64, n_layers=2, k=8, pattern="SF")
    layers = synth.make_layers(wl)
    with pytest.raises(ic.NoCachedIndices):
        _run_stack(ic, wl, layers, pattern="SF")


def test_stack_decode_rows_match_oracle(ic):
    wl = synth.Workload("decode_small", 4, 1, 32768, 4, 64, 128, 2048, 16, 128, "FSSS", 32767, 25)
    layers = synth.make_layers(wl)
    st = _run_stack(ic, wl, layers)
    check_idx_valid(st.idx_cache, wl.q_offset, wl.k)
    _compare_stack(st, wl, layers, None)


def test_stack_prefill_8k_full_size_sampled_rows(ic):
    """The benchmarked configuration at full size: every row checked for
    validity on the device, a bounded sample of rows against the oracle."""
    wl = synth.WORKLOADS["prefill_8k"]
    layers = synth.make_layers(wl, indexer_for_all=False)
    st = _run_stack(ic, wl, layers)
    for l in range(wl.n_layers):
        check_idx_valid(st.dumps[l], 0, wl.k)
    rows = synth.sample_rows(wl, 40)
    _compare_stack(st, wl, layers, rows)
