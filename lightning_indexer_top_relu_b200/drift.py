"""Drift-triggered index refresh: a dynamic F/S schedule.

IndexCache fixes the F/S pattern offline.  The kualia.ai review of the paper
(Conclusion) asks whether sharing should instead be decided at run time:
reuse a neighbour's indices while they remain a good proxy and refresh only
when they have drifted.  This module is that policy, built from the library's
existing calls:

* an F layer of the base pattern runs as always (indexer + top-k overwrite
  the index cache, then attention);
* an S layer first runs a probe: its own indexer and top-k on the last
  `probe_rows` query rows of each sequence (a fraction probe_rows / Lq of an
  F layer's indexer work), and the overlap |A & B| / k of those rows' fresh
  top-k with the cached rows (ic_index_overlap).  If the mean overlap over
  probe rows with t >= k falls below `tau`, the layer is promoted to F (full
  indexer + top-k refresh the cache); otherwise it attends over the cache.

A layer promoted this way needs its indexer inputs, which a static IndexCache
model would have dropped.  Reading the overlap back to the host costs one
synchronisation per S layer.  Leading S layers are an error, as in the static
stack.
"""
from __future__ import annotations

import ctypes
from typing import List, Optional, Sequence

import numpy as np


class DriftRefreshStack:
    """Runs a base F/S pattern with drift-triggered refresh.

    backend: an object with
      full_layer(l)             indexer + top-k of layer l into the cache, then attention
      shared_layer(l)           attention of layer l over the cache
      probe(l, n_rows)          (counts [m, 3], t [m]): |A&B|, |A|, |B| of layer l's own
                                top-k against the cache on the last n_rows rows of each
                                sequence, and those rows' positions
      outputs()                 per-layer outputs
    """

    def __init__(self, base_pattern: str, backend, k: int, tau: float = 0.7,
                 probe_rows: int = 128):
        if not 0.0 <= tau <= 1.0:
            raise ValueError("tau must lie in [0, 1]")
        self.base = base_pattern
        self.backend = backend
        self.k = k
        self.tau = tau
        self.probe_rows = probe_rows
        self.run_pattern = ""
        self.overlaps: List[Optional[float]] = []

    def forward(self):
        run, overlaps = [], []
        for l, c in enumerate(self.base):
            if c in "F1":
                self.backend.full_layer(l)
                run.append("F")
                overlaps.append(None)
                continue
            if c not in "S0":
                raise ValueError(f"pattern character {c!r} is neither F/1 nor S/0")
            if not run:
                raise ValueError("the base pattern starts with a shared layer; the index cache "
                                 "stays empty until a full layer has run")
            counts, t = self.backend.probe(l, self.probe_rows)
            keep = np.asarray(t) >= self.k
            ov = float(np.mean(np.asarray(counts)[keep, 0] / self.k)) if keep.any() else 1.0
            overlaps.append(ov)
            if ov < self.tau:
                self.backend.full_layer(l)
                run.append("F")
            else:
                self.backend.shared_layer(l)
                run.append("S")
        self.run_pattern = "".join(run)
        self.overlaps = overlaps
        return self.backend.outputs()


class GpuBackend:
    """The library's calls on this process's GPU: one index cache and one
    workspace shared by every layer; layers as in LayerStack (dicts of CUDA
    tensors, indexer inputs present on every layer that may run as F)."""

    def __init__(self, layers: Sequence[dict], dims, stream=None, rows_per_chunk: int = 0):
        import torch
        from . import indexcache as ic
        self.ic, self.torch = ic, torch
        self.layers = list(layers)
        self.dims = dims
        self.stream = stream
        dev = layers[0]["q"].device
        d = dims
        self.idx_cache = torch.empty(d.B, d.Lq, d.k, device=dev, dtype=torch.int32)
        self.outs = [torch.empty_like(L["q"]) for L in layers]
        nbytes = max(ic.layer_stack_workspace_bytes(d, 1, rows_per_chunk),
                     ic.sparse_attn_unique_workspace_bytes(d.B, d.Lq, d.Lk, d.q_offset, d.Hq, d.d,
                                                           d.k))
        self.ws = torch.empty(max(int(nbytes), 16), device=dev, dtype=torch.uint8)

    def _table(self, l):
        ic, L = self.ic, self.layers[l]
        t = (ic.ICLayer * 1)()
        t[0] = ic.ICLayer(ic._ptr(L["q"]), ic._ptr(L["k"]), ic._ptr(L["v"]), ic._ptr(L["q_idx"]),
                          ic._ptr(L["k_idx"]), ic._ptr(L["w"]), ic._ptr(self.outs[l]), None, None)
        return t

    def full_layer(self, l):
        ic = self.ic
        rc = ic.lib().ic_layer_stack_forward(b"F", 1, self._table(l), ctypes.byref(self.dims),
                                             ic._ptr(self.idx_cache), ic._ptr(self.ws),
                                             self.ws.numel(), ic._stream(self.stream))
        ic._check(rc, "ic_layer_stack_forward (refresh)")

    def shared_layer(self, l):
        L = self.layers[l]
        self.ic.sparse_attn_unique(L["q"], L["k"], L["v"], self.idx_cache, self.dims.q_offset,
                                   self.dims.scale, out=self.outs[l], want_lse=False, ws=self.ws,
                                   stream=self.stream)

    def probe(self, l, n_rows):
        d, L, torch = self.dims, self.layers[l], self.torch
        p = min(int(n_rows), d.Lq)
        i0 = d.Lq - p
        # The slices are copied and the counts read back on the backend's
        # stream, so they are ordered after the layers already enqueued there
        # (the copy of the cache waits for the last F layer's top-k, the read
        # waits for the overlap kernel).
        st = self.stream if self.stream is not None else torch.cuda.current_stream()
        with torch.cuda.stream(st):
            q_idx = L["q_idx"][:, i0:].contiguous()
            w = L["w"][:, i0:].contiguous()
            sc = self.ic.indexer_scores(q_idx, L["k_idx"], w, d.q_offset + i0, stream=st)
            pidx = self.ic.topk_select(sc, d.k, d.q_offset + i0, stream=st)
            cached = self.idx_cache[:, i0:].contiguous()
            counts = self.ic.index_overlap(pidx, cached, d.Lk, stream=st)
            host = counts.cpu()                     # on st: waits for the overlap kernel
        t = np.tile(np.arange(i0, d.Lq) + d.q_offset, d.B)
        return host.numpy(), t                                          # host sync

    def outputs(self):
        return self.outs
