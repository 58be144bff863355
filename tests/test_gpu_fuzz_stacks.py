"""Seeded random layer stacks through the whole path against the oracle.

Each case draws, from a fixed seed, one small configuration inside the
library's supported set (batch, ragged query count, continuation offset,
indexer heads and width, k, attention heads and head dim, an F-first layer
pattern) and runs ic_layer_stack_forward over it twice, with the indexer ->
top-k fusion forced off and on.  Bars: every index row valid; each F layer's
rows bit-exact against the oracle's sort-based top-k of the GPU's own
indexer scores (the top-k parity rule); every S layer's rows bitwise equal to
its F layer's; mean top-k set overlap >= 0.99 against the oracle's own
scores and attention within 2e-2 on the rows whose sets agree (the
layer-stack bars of test_gpu_parity); fused and plain runs identical.
"""
import numpy as np
import pytest
import torch

import oracle
from lightning_indexer_top_relu_b200 import build, synth
from test_gpu_parity import _compare_stack, _cuda, check_idx_valid

N_CASES = 64


def draw_case(seed: int) -> dict:
    """One configuration from the supported set (host-side, no device use)."""
    rng = np.random.default_rng(9000 + seed)
    B = int(rng.integers(1, 4))
    Lq = int(rng.choice([1, int(rng.integers(2, 130)), int(rng.integers(130, 700))]))
    if Lq == 1:                                   # decode rows deep in a sequence
        q_offset = int(rng.integers(0, 3000))
    else:                                         # prefill, or a continuation chunk
        q_offset = int(rng.choice([0, 0, int(rng.integers(1, 600))]))
    Lk = Lq + q_offset
    H_I = int(rng.choice([4, 8, 16, 32, 64, 128]))
    d_I = int(rng.choice([64, 128]))
    Hq = int(rng.choice([8, 16]))
    d = int(rng.choice([64, 128]))
    k = int(min(Lk, rng.choice([int(rng.integers(1, 8)), int(rng.integers(8, 64)),
                                int(rng.integers(64, 300))])))
    n_layers = int(rng.integers(1, 5))
    pattern = "F" + "".join(rng.choice(["F", "S", "S"], n_layers - 1))
    return dict(B=B, Lq=Lq, Lk=Lk, q_offset=q_offset, H_I=H_I, d_I=d_I, Hq=Hq, d=d, k=k,
                n_layers=n_layers, pattern=pattern, cfg_id=400 + seed)


def test_case_draws_stay_in_the_supported_set():
    # host-only check of the generator itself
    for s in range(N_CASES):
        c = draw_case(s)
        assert 1 <= c["k"] <= c["Lk"] and c["q_offset"] + c["Lq"] <= c["Lk"]
        assert c["pattern"][0] == "F" and len(c["pattern"]) == c["n_layers"]


@pytest.fixture(scope="module")
def ic():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    from lightning_indexer_top_relu_b200 import indexcache
    return indexcache


def _stack(ic, wl, layers, fused):
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    st = ic.LayerStack(wl.pattern, [_cuda(L) for L in layers], dims, want_lse=True,
                       dump_idx=True, fused_topk=fused)
    st.forward()
    torch.cuda.synchronize()
    assert ic.get_last_device_error() == 0
    return st


@pytest.mark.gpu
@pytest.mark.parametrize("seed", range(N_CASES))
def test_random_stack_matches_oracle(ic, seed):
    c = draw_case(seed)
    wl = synth.custom(B=c["B"], Lq=c["Lq"], Lk=c["Lk"], q_offset=c["q_offset"], n_layers=c["n_layers"],
                      H_I=c["H_I"], d_I=c["d_I"], k=c["k"], Hq=c["Hq"], d=c["d"],
                      pattern=c["pattern"], cfg_id=c["cfg_id"])
    layers = synth.make_layers(wl)
    plain = _stack(ic, wl, layers, 0)
    fused = _stack(ic, wl, layers, 1)
    check_idx_valid(plain.idx_cache, wl.q_offset, wl.k)
    for l in range(wl.n_layers):
        assert torch.equal(plain.dumps[l], fused.dumps[l]), (c, l)
        assert torch.equal(plain.outs[l], fused.outs[l]), (c, l)
        if wl.pattern[l] == "F":
            L = _cuda(layers[l])
            sc = ic.indexer_scores(L["q_idx"], L["k_idx"], L["w"], wl.q_offset)
            want = oracle.topk_sort(sc.reshape(-1, wl.Lk).cpu().numpy(),
                                    oracle.row_positions(wl.B, wl.Lq, wl.q_offset), wl.k)
            assert np.array_equal(plain.dumps[l].cpu().numpy().reshape(-1, wl.k), want), (c, l)
    # at most 96 rows through the oracle keeps each case to seconds
    n = wl.B * wl.Lq
    rows = None if n <= 96 else np.sort(np.random.default_rng(seed).choice(n, 96, replace=False))
    _compare_stack(plain, wl, layers, rows)
