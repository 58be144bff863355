"""Drift-triggered refresh on CPU: the policy of
DriftRefreshStack driven by an oracle backend.  Its outputs must equal the
static oracle stack run with the F/S pattern the policy chose, and the policy
must refresh exactly the layers whose own top-k has drifted from the cache."""
import numpy as np
import pytest

import oracle
from lightning_indexer_top_relu_b200 import synth
from lightning_indexer_top_relu_b200.drift import DriftRefreshStack


class OracleBackend:
    """The backend's steps on the CPU oracle."""

    def __init__(self, layers, k, q_offset=0):
        self.layers, self.k, self.q_offset = list(layers), k, q_offset
        qi = oracle._bf16_bits(self.layers[0]["q"])
        self.B, self.Lq = qi.shape[0], qi.shape[1]
        self.Lk = oracle._bf16_bits(self.layers[0]["k"]).shape[1]
        self.cache = None
        self.outs = [None] * len(layers)

    def _topk(self, L, rows):
        sc = oracle.indexer_scores(L["q_idx"], L["k_idx"], L["w"], self.q_offset, rows)
        tpos = oracle.row_positions(self.B, self.Lq, self.q_offset, rows)
        return oracle.topk_sort(sc.astype(np.float32), tpos, self.k)

    def full_layer(self, l):
        L = self.layers[l]
        self.cache = self._topk(L, None)
        self.outs[l] = oracle.sparse_attn(L["q"], L["k"], L["v"], self.cache, self.q_offset)[0]

    def shared_layer(self, l):
        L = self.layers[l]
        self.outs[l] = oracle.sparse_attn(L["q"], L["k"], L["v"], self.cache, self.q_offset)[0]

    def probe(self, l, n_rows):
        p = min(int(n_rows), self.Lq)
        rows = [b * self.Lq + i for b in range(self.B) for i in range(self.Lq - p, self.Lq)]
        fresh = self._topk(self.layers[l], rows)
        counts = oracle.index_overlap(fresh, self.cache[rows], self.Lk)
        return counts, oracle.row_positions(self.B, self.Lq, self.q_offset, rows)

    def outputs(self):
        return self.outs


WL = synth.Workload("drift", 1, 512, 512, 4, 8, 64, 64, 8, 64, "FSSS", 0, 13, True)


def _layers(replace=()):
    """Correlated layers; the layers in `replace` get indexer inputs of an
    unrelated draw (their own top-k then shares little with layer 0's)."""
    layers = synth.make_layers(WL)
    other = synth.make_layers(synth.custom(Lq=WL.Lq, n_layers=WL.n_layers, H_I=WL.H_I,
                                           d_I=WL.d_I, k=WL.k, Hq=WL.Hq, d=WL.d, cfg_id=41))
    for l in replace:
        for n in ("q_idx", "k_idx", "w"):
            layers[l][n] = other[l][n]
    return layers


def _run(layers, tau, probe_rows=64):
    st = DriftRefreshStack(WL.pattern, OracleBackend(layers, WL.k), WL.k, tau, probe_rows)
    outs = st.forward()
    ref, _, _ = oracle.layer_stack(st.run_pattern, layers, WL.k)
    for l in range(WL.n_layers):
        assert np.array_equal(outs[l], ref[l])            # same arithmetic as the static stack
    return st


def test_correlated_layers_keep_the_static_pattern():
    st = _run(_layers(), tau=0.5)
    assert st.run_pattern == "FSSS"
    assert all(ov > 0.5 for ov in st.overlaps[1:])


def test_a_drifted_layer_is_refreshed():
    st = _run(_layers(replace=(2,)), tau=0.5)
    # layer 2 (an unrelated draw) refreshes the cache; layer 3, correlated
    # with layers 0 and 1, then differs from that refreshed cache and refreshes too
    assert st.run_pattern == "FSFF"
    assert st.overlaps[1] > 0.5 and st.overlaps[2] < 0.5 and st.overlaps[3] < 0.5


def test_tau_one_refreshes_every_shared_layer_and_zero_none():
    assert _run(_layers(), tau=1.0).run_pattern == "FFFF"
    assert _run(_layers(replace=(1, 2, 3)), tau=0.0).run_pattern == "FSSS"


def test_probe_rows_that_select_everything_never_trigger():
    # the first 64 rows select every visible position (t < k): no drift to see
    layers = _layers(replace=(1,))
    b = OracleBackend(layers, WL.k)
    st = DriftRefreshStack(WL.pattern, b, WL.k, tau=0.99, probe_rows=64)
    b.probe = lambda l, n: (np.zeros((4, 3), np.int32), np.arange(4))    # t < k only
    st.forward()
    assert st.run_pattern == "FSSS" and st.overlaps[1:] == [1.0, 1.0, 1.0]


def test_leading_shared_layer_is_an_error():
    st = DriftRefreshStack("SFSS", OracleBackend(_layers(), WL.k), WL.k, 0.5)
    with pytest.raises(ValueError):
        st.forward()
