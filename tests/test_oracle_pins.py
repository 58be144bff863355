"""Pins for the CPU oracle: values and properties fixed by the pages or by
mathematics, never by the oracle itself and never by the CUDA path.

Each test below is chosen so that a plausible slip in the oracle (a dropped
ReLU, a swapped t/s index, a transposed operand, a wrong tie rule, a missing
causal mask, a wrong softmax normaliser) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from lightning_indexer_top_relu_b200 import synth


def _bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _num(x):
    if isinstance(x, str):
        return {"-inf": -math.inf, "ln 3": math.log(3.0), "ln 4": math.log(4.0)}[x]
    return float(x)


# ------------------------------------------------------------------ indexer

def test_indexer_hand_worked_example(golden_dir):
    g = _load(golden_dir, "indexer_hand_example.json")
    q = _bf16(g["q_idx"])[None]          # [1, 3, 2, 2]
    k = _bf16(g["k_idx"])[None]          # [1, 3, 2]
    w = torch.tensor(g["w"], dtype=torch.float32)[None]
    sc = oracle.indexer_scores(q, k, w)
    want = np.array([[_num(x) for x in row] for row in g["scores"]])
    assert np.array_equal(sc, want)
    idx = oracle.topk_sort(sc.astype(np.float32), oracle.row_positions(1, 3, 0), g["k"])
    assert idx.tolist() == g["topk"]


def test_indexer_nonnegative_dots_reduce_to_matvec():
    """With every q_I . k_I >= 0 the ReLU is the identity, so the score is the
    single dot product k_I[s] . (sum_j w_j q_I[t,j]) (a plain matvec)."""
    rng = np.random.default_rng(1)
    B, L, H, dI = 2, 37, 3, 16
    q = _bf16(rng.uniform(0, 1, (B, L, H, dI)))
    k = _bf16(rng.uniform(0, 1, (B, L, dI)))
    w = torch.tensor(rng.normal(size=(B, L, H)), dtype=torch.float32)
    sc = oracle.indexer_scores(q, k, w).reshape(B, L, L)
    qd, kd, wd = q.double().numpy(), k.double().numpy(), w.double().numpy()
    for b in range(B):
        for t in range(L):
            v = (wd[b, t][:, None] * qd[b, t]).sum(0)
            want = kd[b] @ v
            assert np.allclose(sc[b, t, : t + 1], want[: t + 1], rtol=1e-12, atol=1e-12)
            assert np.all(np.isneginf(sc[b, t, t + 1:]))


def test_indexer_matches_a_library_evaluation_of_the_formula():
    """Mixed-sign q_I, k_I and w, B > 1, a row offset: the score equals an
    fp64 torch evaluation of sum_j w[t,j] * relu(q_I[t,j] . k_I[s]) for
    s <= t (an independent routine: einsum, clamp, a weighted head sum)."""
    rng = np.random.default_rng(9)
    B, Lq, Lk, H, dI, q0 = 2, 23, 40, 5, 16, 17
    q = _bf16(rng.normal(size=(B, Lq, H, dI)))
    k = _bf16(rng.normal(size=(B, Lk, dI)))
    w = torch.tensor(rng.normal(size=(B, Lq, H)), dtype=torch.float32)
    sc = oracle.indexer_scores(q, k, w, q_offset=q0).reshape(B, Lq, Lk)
    dots = torch.einsum("bthc,bsc->bths", q.double(), k.double())
    ref = (w.double()[..., None] * dots.clamp(min=0)).sum(dim=2).numpy()
    t = np.arange(Lq)[:, None] + q0
    vis = np.arange(Lk)[None, :] <= t
    assert np.allclose(sc[:, vis], ref[:, vis], rtol=1e-12, atol=1e-12)
    assert np.all(np.isneginf(sc[:, ~vis]))


def test_indexer_negative_dots_give_zero():
    """Every q_I . k_I < 0 -> every visible score is exactly 0 (ReLU clips)."""
    rng = np.random.default_rng(2)
    q = _bf16(rng.uniform(0.1, 1, (1, 20, 4, 8)))
    k = _bf16(-rng.uniform(0.1, 1, (1, 20, 8)))
    w = torch.tensor(rng.normal(size=(1, 20, 4)), dtype=torch.float32)
    sc = oracle.indexer_scores(q, k, w).reshape(20, 20)
    tri = np.tril(np.ones((20, 20), dtype=bool))
    assert np.all(sc[tri] == 0.0)
    assert np.all(np.isneginf(sc[~tri]))


def test_indexer_relu_keeps_sign_per_head():
    """One head, one dim: score = w * max(0, q*k) elementwise (closed form)."""
    qv = np.array([2.0, -1.0, 0.5, -3.0, 1.0])
    kv = np.array([1.0, -2.0, 4.0, 0.25, -1.0])
    wv = np.array([1.5, -2.0, 0.5, 1.0, 3.0])
    sc = oracle.indexer_scores(_bf16(qv.reshape(1, 5, 1, 1)), _bf16(kv.reshape(1, 5, 1)),
                               torch.tensor(wv.reshape(1, 5, 1), dtype=torch.float32))
    for t in range(5):
        for s in range(5):
            want = wv[t] * max(0.0, qv[t] * kv[s]) if s <= t else -math.inf
            assert sc[t, s] == want


def test_indexer_invariants_head_permutation_and_scaling():
    rng = np.random.default_rng(3)
    q = _bf16(rng.normal(size=(1, 30, 5, 8)))
    k = _bf16(rng.normal(size=(1, 30, 8)))
    w = torch.tensor(rng.normal(size=(1, 30, 5)), dtype=torch.float32)
    base = oracle.indexer_scores(q, k, w)
    perm = [3, 0, 4, 1, 2]
    assert np.allclose(oracle.indexer_scores(q[:, :, perm], k, w[:, :, perm]), base, rtol=1e-13)
    assert np.array_equal(oracle.indexer_scores(q, k, 2 * w), 2 * base)


def test_indexer_row_sampling_matches_full():
    wl = synth.custom(Lq=70, H_I=2, d_I=64, k=8, Hq=2, d=64)
    L = synth.make_layers(wl)[0]
    full = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"])
    rows = [0, 5, 69, 33]
    part = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"], rows=rows)
    assert np.array_equal(part, full[rows])


# ------------------------------------------------------------------ top-k

@pytest.mark.parametrize("draw", ["ties", "gauss", "signed_zero"])
def test_topk_sort_equals_bruteforce_count(draw):
    rng = np.random.default_rng({"ties": 4, "gauss": 5, "signed_zero": 6}[draw])
    n, Lk = 300, 60
    if draw == "ties":
        sc = rng.integers(-1, 2, size=(n, Lk)).astype(np.float32)
    elif draw == "gauss":
        sc = rng.normal(size=(n, Lk)).astype(np.float32)
    else:
        sc = np.where(rng.random((n, Lk)) < 0.5, np.float32(-0.0), np.float32(0.0))
        sc[:, ::7] = 1.0
    tpos = rng.integers(0, Lk + 10, size=n)  # includes t >= Lk (all positions visible)
    for k in (1, 5, 17, 60, 80):
        a = oracle.topk_sort(sc, tpos, k)
        b = oracle.topk_count(sc, tpos, k)
        assert np.array_equal(a, b), (draw, k)


def test_topk_matches_stable_argsort():
    """A stable library sort on (-score) orders ties by position, which is the
    tie rule; its first min(k, t+1) entries, sorted, are the selection."""
    rng = np.random.default_rng(7)
    n, Lk, k = 200, 90, 13
    sc = rng.integers(-3, 4, size=(n, Lk)).astype(np.float32)
    sc[::3] = rng.normal(size=(len(sc[::3]), Lk)).astype(np.float32)
    tpos = rng.integers(0, Lk, size=n)
    got = oracle.topk_sort(sc, tpos, k)
    for r in range(n):
        vis = sc[r, : tpos[r] + 1]
        order = np.argsort(-vis, kind="stable")[: min(k, len(vis))]
        want = np.full(k, -1)
        want[: len(order)] = np.sort(order)
        assert np.array_equal(got[r], want)


def test_topk_all_ties_closed_form():
    """w = 0 makes every score 0, so the tie rule alone decides:
    idx = [0, 1, ..., min(k, t+1)-1] then -1 padding."""
    wl = synth.custom(Lq=50, H_I=3, d_I=64, k=8)
    L = synth.make_layers(wl)[0]
    sc = oracle.indexer_scores(L["q_idx"], L["k_idx"], torch.zeros_like(L["w"]))
    idx = oracle.topk_sort(sc.astype(np.float32), oracle.row_positions(1, 50, 0), 8)
    for t in range(50):
        m = min(8, t + 1)
        assert idx[t].tolist() == list(range(m)) + [-1] * (8 - m)


def test_topk_increasing_scores_closed_form():
    """q_I = e0, k_I[s] = (s/64) e0, w = 1: the score grows with s, so the
    selection is the last min(k, t+1) visible positions."""
    L, dI, k = 64, 64, 10
    q = np.zeros((1, L, 1, dI)); q[..., 0] = 1.0
    kk = np.zeros((1, L, dI)); kk[0, :, 0] = np.arange(L) / 64.0
    sc = oracle.indexer_scores(_bf16(q), _bf16(kk), torch.ones(1, L, 1))
    idx = oracle.topk_sort(sc.astype(np.float32), oracle.row_positions(1, L, 0), k)
    for t in range(L):
        m = min(k, t + 1)
        assert idx[t].tolist() == list(range(t - m + 1, t + 1)) + [-1] * (k - m)


# ------------------------------------------------------------------ attention

def test_attention_hand_worked_example(golden_dir):
    g = _load(golden_dir, "attn_hand_example.json")
    q = _bf16(g["q"]).reshape(1, 1, 1, 2)
    K = _bf16(g["K"]).reshape(1, 3, 1, 2)
    V = _bf16(g["V"]).reshape(1, 3, 1, 2)
    idx = np.array([g["idx"]], dtype=np.int32)
    out, lse = oracle.sparse_attn(q, K, V, idx, q_offset=g["t"], scale=_num(g["scale"]))
    assert np.allclose(out[0, 0], g["out"][0], rtol=0, atol=1e-12)
    assert abs(lse[0, 0] - _num(g["lse"][0])) < 1e-12


def test_sparse_equals_dense_and_library_sdpa_when_k_ge_L():
    """k >= L selects every visible position, so sparse attention must equal
    causal dense attention, which a library routine computes independently."""
    wl = synth.custom(B=2, Lq=40, H_I=2, d_I=64, k=64, Hq=4, d=64)
    L = synth.make_layers(wl)[0]
    sc = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"])
    idx = oracle.topk_sort(sc.astype(np.float32), oracle.row_positions(2, 40, 0), 64)
    sp, sp_lse = oracle.sparse_attn(L["q"], L["k"], L["v"], idx)
    de, de_lse = oracle.dense_attn(L["q"], L["k"], L["v"])
    assert np.allclose(sp, de, rtol=0, atol=1e-13)
    assert np.allclose(sp_lse, de_lse, rtol=0, atol=1e-13)
    q = L["q"].double().transpose(1, 2)                   # [B, Hq, L, d]
    K = L["k"].double().transpose(1, 2).expand(-1, 4, -1, -1)
    V = L["v"].double().transpose(1, 2).expand(-1, 4, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, is_causal=True)
    ref = ref.transpose(1, 2).reshape(80, 4, 64).numpy()
    assert np.allclose(sp, ref, rtol=0, atol=1e-12)


def test_attention_constant_values():
    """Every gathered V row equal to c -> the output is c whatever the weights."""
    rng = np.random.default_rng(8)
    q = _bf16(rng.normal(size=(1, 16, 3, 8)))
    K = _bf16(rng.normal(size=(1, 16, 1, 8)))
    c = rng.normal(size=8)
    V = _bf16(np.broadcast_to(c, (1, 16, 1, 8)))
    idx = np.stack([np.sort(rng.choice(t + 1, size=min(4, t + 1), replace=False)).tolist()
                    + [-1] * (4 - min(4, t + 1)) for t in range(16)]).astype(np.int32)
    out, _ = oracle.sparse_attn(q, K, V, idx)
    cb = V[0, 0, 0].double().numpy()
    assert np.allclose(out, np.broadcast_to(cb, out.shape), rtol=0, atol=1e-12)


def test_attention_dominant_logit_picks_its_value_row():
    d = 8
    q = np.zeros((1, 1, 1, d)); q[..., 0] = 1.0
    K = np.zeros((1, 6, 1, d)); K[0, 4, 0, 0] = 64.0      # z = 64 vs 0 elsewhere (scale 1)
    V = np.arange(6 * d, dtype=np.float64).reshape(1, 6, 1, d)
    out, lse = oracle.sparse_attn(_bf16(q), _bf16(K), _bf16(V),
                                  np.array([[0, 2, 4, 5]], dtype=np.int32), q_offset=5, scale=1.0)
    assert np.allclose(out[0, 0], V[0, 4, 0], atol=1e-20 + 1e-24)
    assert abs(lse[0, 0] - (64.0 + math.log1p(3 * math.exp(-64.0)))) < 1e-12


def test_attention_row_sampling_matches_full():
    """Row r of a sampled call is flattened row rows[r] of the full call, and
    it reads index row r (one index row per requested row)."""
    wl = synth.custom(B=2, Lq=30, Lk=50, q_offset=20, H_I=2, d_I=64, k=8, Hq=3, d=64)
    L = synth.make_layers(wl)[0]
    sc = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"], q_offset=20)
    idx = oracle.topk_sort(sc.astype(np.float32), oracle.row_positions(2, 30, 20), 8)
    full, full_lse = oracle.sparse_attn(L["q"], L["k"], L["v"], idx, q_offset=20)
    dense, dense_lse = oracle.dense_attn(L["q"], L["k"], L["v"], q_offset=20)
    rows = [59, 0, 31, 7, 30]
    part, part_lse = oracle.sparse_attn(L["q"], L["k"], L["v"], idx[rows], q_offset=20, rows=rows)
    assert np.array_equal(part, full[rows]) and np.array_equal(part_lse, full_lse[rows])
    dpart, dpart_lse = oracle.dense_attn(L["q"], L["k"], L["v"], q_offset=20, rows=rows)
    assert np.array_equal(dpart, dense[rows]) and np.array_equal(dpart_lse, dense_lse[rows])


def test_attention_empty_row_and_out_of_range_index():
    q = _bf16(np.ones((1, 1, 2, 4)))
    K = _bf16(np.ones((1, 3, 1, 4)))
    V = _bf16(np.ones((1, 3, 1, 4)))
    out, lse = oracle.sparse_attn(q, K, V, np.array([[-1, -1]], dtype=np.int32), q_offset=2)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    with pytest.raises(ValueError):   # index beyond the visible range t
        oracle.sparse_attn(q, K, V, np.array([[0, 2]], dtype=np.int32), q_offset=1)


def test_queries_past_the_last_key_are_rejected():
    """q_offset + Lq > Lk puts a query after the last key; the library
    rejects that before any launch, and so does every oracle step (it used to
    clamp t to Lk - 1 silently)."""
    wl = synth.custom(Lq=4, Lk=6, q_offset=2, H_I=2, d_I=64, k=4, Hq=2, d=64)
    L = synth.make_layers(wl)[0]
    idx = np.zeros((4, 4), dtype=np.int32)
    oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"], q_offset=2)        # t <= 5: fine
    oracle.sparse_attn(L["q"], L["k"], L["v"], idx, q_offset=2)
    oracle.dense_attn(L["q"], L["k"], L["v"], q_offset=2)
    with pytest.raises(ValueError):
        oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"], q_offset=3)
    with pytest.raises(ValueError):
        oracle.sparse_attn(L["q"], L["k"], L["v"], idx, q_offset=3)
    with pytest.raises(ValueError):
        oracle.dense_attn(L["q"], L["k"], L["v"], q_offset=3)


# ------------------------------------------------------------------ layer stack (a3, a5)

def _check_idx_valid(idx, tpos, k):
    for r, t in enumerate(tpos):
        row = idx[r]
        m = min(k, t + 1)
        assert np.all(row[:m] >= 0) and np.all(row[:m] <= t)
        assert np.all(np.diff(row[:m]) > 0)
        assert np.all(row[m:] == -1)


def test_stack_shared_layers_reuse_nearest_full_layer():
    wl = synth.custom(Lq=96, n_layers=6, H_I=2, d_I=64, k=16, Hq=2, d=64, pattern="FSSFSS")
    layers = synth.make_layers(wl)
    outs, idxs, _ = oracle.layer_stack(wl.pattern, layers, wl.k)
    assert idxs[1] is idxs[0] and idxs[2] is idxs[0]
    assert idxs[4] is idxs[3] and idxs[5] is idxs[3]
    assert not np.array_equal(idxs[0], idxs[3])
    tpos = oracle.row_positions(1, 96, 0)
    for l in (0, 3):
        _check_idx_valid(idxs[l], tpos, wl.k)
    # '1'/'0' spells the same pattern
    outs2, idxs2, _ = oracle.layer_stack("100100", layers, wl.k)
    for a, b in zip(outs, outs2):
        assert np.array_equal(a, b)
    # An S layer attends exactly like an F layer handed the cached indices.
    o2, _ = oracle.sparse_attn(layers[2]["q"], layers[2]["k"], layers[2]["v"], idxs[0])
    assert np.array_equal(o2, outs[2])


def test_stack_on_sampled_rows_equals_the_full_stack_there():
    """The layer loop on a row sample (what the full-size checks use) gives,
    row for row, the full run's indices, outputs and log-sum-exps."""
    wl = synth.custom(B=2, Lq=40, Lk=60, q_offset=20, n_layers=3, H_I=2, d_I=64, k=8, Hq=2,
                      d=64, pattern="FSF")
    layers = synth.make_layers(wl)
    outs, idxs, lses = oracle.layer_stack(wl.pattern, layers, wl.k, q_offset=20)
    rows = [79, 3, 40, 0, 55]
    o2, i2, l2 = oracle.layer_stack(wl.pattern, layers, wl.k, q_offset=20, rows=rows)
    for l in range(3):
        assert np.array_equal(i2[l], idxs[l][rows])
        assert np.array_equal(o2[l], outs[l][rows])
        assert np.array_equal(l2[l], lses[l][rows])


def test_stack_leading_shared_layer_is_an_error():
    wl = synth.custom(Lq=8, n_layers=2, k=4, pattern="SF")
    layers = synth.make_layers(wl)
    with pytest.raises(oracle.NoCachedIndices):
        oracle.layer_stack("SF", layers, 4)
    with pytest.raises(ValueError):
        oracle.layer_stack("FX", layers, 4)


def test_stack_no_state_across_calls():
    """The cache lives inside one call: a second sequence never sees the
    first one's indices (skill page, Common Pitfalls)."""
    wl = synth.custom(Lq=32, n_layers=2, H_I=2, d_I=64, k=8, pattern="FS")
    a = synth.make_layers(wl)
    wl2 = synth.custom(Lq=32, n_layers=2, H_I=2, d_I=64, k=8, pattern="FS", cfg_id=11)
    b = synth.make_layers(wl2)
    _, ia, _ = oracle.layer_stack("FS", a, 8)
    _, ib, _ = oracle.layer_stack("FS", b, 8)
    _, ia2, _ = oracle.layer_stack("FS", a, 8)
    assert np.array_equal(ia[1], ia2[1]) and not np.array_equal(ia[1], ib[1])


def test_decode_row_sees_whole_cache():
    """Decode: one query per sequence at q_offset = Lk-1 sees all Lk positions."""
    wl = synth.custom(B=3, Lq=1, Lk=40, q_offset=39, H_I=2, d_I=64, k=8, Hq=2, d=64)
    L = synth.make_layers(wl)[0]
    sc = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"], q_offset=39)
    assert np.all(np.isfinite(sc))
    idx = oracle.topk_sort(sc.astype(np.float32), oracle.row_positions(3, 1, 39), 8)
    _check_idx_valid(idx, [39, 39, 39], 8)


def test_synthetic_layers_overlap_in_the_reported_band():
    """Adjacent synthetic layers share a large part of their top-k, as the
    pages report for real models (70-100%); checked on a smaller shape."""
    wl = synth.Workload("ov", 1, 1024, 1024, 2, 8, 64, 128, 2, 64, "FF", 0, 12, True)
    layers = synth.make_layers(wl)
    rows = list(range(600, 1024, 16))
    tpos = oracle.row_positions(1, 1024, 0, rows)
    ids = []
    for L in layers:
        sc = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"], rows=rows)
        ids.append(oracle.topk_sort(sc.astype(np.float32), tpos, 128))
    ov = [len(set(a) & set(b)) / 128 for a, b in zip(ids[0], ids[1])]
    assert 0.6 <= np.mean(ov) <= 1.0


# ------------------------------------------------------------------ cross-layer overlap (f2)

def test_overlap_hand_example():
    # A = {0, 3, 5, 9}, B = {3, 4, 5} (+ holes): |A&B| = 2, |A| = 4, |B| = 3,
    # overlap 2/4, Jaccard 2/5
    a = np.array([[0, 3, 5, 9]], dtype=np.int32)
    b = np.array([[5, -1, 3, 4]], dtype=np.int32)
    c = oracle.index_overlap(a, b, 10)
    assert c.tolist() == [[2, 4, 3]]
    assert oracle.overlap_fraction(c, 4)[0] == 0.5
    assert abs(oracle.jaccard(c)[0] - 0.4) < 1e-9
    # a short row (t + 1 < k: holes at the tail): the fraction is still over
    # the k slots of the cache, A = {1, 2}, B = {2, 3, 7} -> 1/4
    c = oracle.index_overlap(np.array([[1, 2, -1, -1]], dtype=np.int32),
                             np.array([[2, 3, 7, -1]], dtype=np.int32), 10)
    assert c.tolist() == [[1, 2, 3]]
    assert oracle.overlap_fraction(c, 4)[0] == 0.25
    assert abs(oracle.jaccard(c)[0] - 0.25) < 1e-9


def test_overlap_matches_python_sets_and_is_symmetric():
    rng = np.random.default_rng(7)
    k, Lk, n = 24, 60, 200
    a = rng.integers(-1, Lk, size=(n, k)).astype(np.int32)     # holes and repeats
    b = rng.integers(-1, Lk, size=(n, k)).astype(np.int32)
    c = oracle.index_overlap(a, b, Lk)
    for r in range(n):
        sa, sb = set(a[r]) - {-1}, set(b[r]) - {-1}
        assert c[r].tolist() == [len(sa & sb), len(sa), len(sb)]
    c2 = oracle.index_overlap(b, a, Lk)
    assert np.array_equal(c2[:, 0], c[:, 0]) and np.array_equal(c2[:, 1:], c[:, 2:0:-1])


def test_overlap_identity_disjoint_and_bad_entries():
    a = np.array([[1, 2, 3], [4, 5, -1]], dtype=np.int32)
    assert oracle.index_overlap(a, a, 8).tolist() == [[3, 3, 3], [2, 2, 2]]
    b = np.array([[5, 6, 7], [0, 1, 2]], dtype=np.int32)
    assert oracle.index_overlap(a, b, 8)[:, 0].tolist() == [0, 0]
    with pytest.raises(ValueError):
        oracle.index_overlap(np.array([[8, 1, 2]], dtype=np.int32), a[:1], 8)
