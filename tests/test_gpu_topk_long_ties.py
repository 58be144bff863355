"""Top-k rows whose k-th score sits in a bin of more than 2048 keys.

The radix select gathers the keys of its threshold bin (the top 11 bits of
the order-preserving key) into a shared-memory candidate list of 2048
entries.  A fuller bin -- long rows of equal or two-valued scores, such as
the all-zero scores that w = 0 produces -- takes full passes over the row
instead.  These cases reach that path (a CPU check below confirms it), with
rows short enough for the shared-memory key cache and rows too long for it,
and compare bit for bit with the oracle like every top-k case.  The stack
case is the method's own degenerate input: with w = 0 every indexer score
is exactly 0, so the tie rule alone decides and the index rows have a
closed form, [0, 1, ..., min(k, t+1) - 1] then -1.
"""
import numpy as np
import pytest
import torch

import oracle
from lightning_indexer_top_relu_b200 import build, synth

CAND_CAPACITY = 2048     # keys of the threshold bin the kernel keeps in shared memory

CASES = [
    # B, Lq, Lk, q_offset, k, draw
    (1, 64, 3000, 2936, 64, "const"),             # every key in one bin
    (1, 64, 5000, 4936, 100, "signed_zeros"),     # +0 and -0 are one key
    (1, 32, 9000, 8968, 2048, "two_values"),      # about 4500 ones hold the k-th key
    (2, 16, 60000, 59984, 2048, "const"),         # rows too long for the key cache
    (1, 3000, 3000, 0, 64, "const"),              # short rows (candidates) and long rows together
]


def _draw(kind, rows, Lk, seed):
    rng = np.random.default_rng(seed)
    if kind == "const":
        return np.full((rows, Lk), -1.5, dtype=np.float32)
    if kind == "signed_zeros":
        return np.where(rng.random((rows, Lk)) < 0.5, np.float32(-0.0), np.float32(0.0))
    if kind == "two_values":
        return rng.integers(0, 2, size=(rows, Lk)).astype(np.float32)
    raise ValueError(kind)


def _threshold_bin_size(row: np.ndarray, k: int) -> int:
    """Keys in the 11-bit bin that holds the row's k-th largest key, for the
    usual order-preserving map of fp32 bits (-0 folded onto +0)."""
    f = np.where(row == 0.0, np.float32(0.0), row).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    key = np.where(u >> 31, (~u) & 0xFFFFFFFF, u | 0x80000000).astype(np.uint64)
    bins = (key >> 21).astype(np.int64)
    kth = np.sort(key)[::-1][min(k, len(key)) - 1]
    return int(np.sum(bins == int(kth >> 21)))


def test_cases_overflow_the_candidate_list():
    """CPU check that each case has rows whose threshold bin exceeds the
    kernel's candidate capacity, so the GPU test below runs the full-pass path."""
    for B, Lq, Lk, q0, k, draw in CASES:
        sc = _draw(draw, B * Lq, Lk, seed=Lk + k)
        t = q0 + Lq - 1                           # the longest row sees t + 1 keys
        n = min(t + 1, Lk)
        assert _threshold_bin_size(sc[-1, :n], k) > CAND_CAPACITY, (B, Lq, Lk, draw)


@pytest.fixture(scope="module")
def ic():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    from lightning_indexer_top_relu_b200 import indexcache
    return indexcache


@pytest.mark.gpu
@pytest.mark.parametrize("B,Lq,Lk,q_offset,k,draw", CASES)
def test_topk_long_tied_rows_bit_exact(ic, B, Lq, Lk, q_offset, k, draw):
    sc = _draw(draw, B * Lq, Lk, seed=Lk + k)
    ref = oracle.topk_sort(sc, oracle.row_positions(B, Lq, q_offset), k)
    gpu = ic.topk_select(torch.from_numpy(sc).reshape(B, Lq, Lk).cuda(), k, q_offset)
    assert np.array_equal(gpu.cpu().numpy().reshape(B * Lq, k), ref)


@pytest.mark.gpu
def test_stack_with_zero_head_weights_keeps_the_first_positions(ic):
    """w = 0: all scores 0, so every row keeps its first min(k, t+1)
    positions; rows t < 6k attend dense-masked, the rest gather, both over
    those positions, and agree with the oracle's attention on them."""
    wl = synth.custom(Lq=3000, n_layers=2, H_I=32, d_I=128, k=64, Hq=16, d=128, pattern="FS",
                      cfg_id=36)
    layers = synth.make_layers(wl)
    for L in layers:
        L["w"] = torch.zeros_like(L["w"])
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    st = ic.LayerStack(wl.pattern, [{n: t.cuda() for n, t in L.items()} for L in layers], dims,
                       want_lse=True, dump_idx=True)
    st.forward()
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    t = np.arange(wl.Lq)
    slot = np.arange(wl.k)
    want = np.where(slot[None, :] < np.minimum(t + 1, wl.k)[:, None], slot[None, :], -1)
    for l in range(2):
        got = st.dumps[l].cpu().numpy().reshape(wl.Lq, wl.k)
        assert np.array_equal(got, want), l
        ref, ref_lse = oracle.sparse_attn(layers[l]["q"], layers[l]["k"], layers[l]["v"],
                                          want.astype(np.int32))
        out = st.outs[l].float().cpu().numpy().reshape(wl.Lq, wl.Hq, wl.d)
        assert np.abs(out - ref).max() <= 2e-2
        lse = st.lses[l].cpu().numpy().reshape(wl.Lq, wl.Hq)
        assert np.abs(lse - ref_lse).max() <= 1e-3
