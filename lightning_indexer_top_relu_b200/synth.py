"""Seeded synthetic inputs for the IndexCache sparse-attention layer stack.

This module draws random tensors and nothing else: it holds none of the
method's arithmetic (no scores, no selection, no attention).  Both the CUDA
path and the CPU oracle are fed from it.

Workloads (named by what they are):

* ``tiny_prefill``  B=1, L=512, 4 layers FSSS, indexer 4 heads x 64, k=64,
  attention 8 query heads / 1 KV head x 64.  Every tensor i.i.d.
  N(0,1)/sqrt(last dim) from one generator seeded 0.
* ``prefill_8k``    B=1, L=8192, 8 layers FSSSFSSS, indexer 32 x 128, k=2048,
  attention 16 / 1 x 128, correlated layers (below).
* ``prefill_64k``   B=1, L=65536, 8 layers, FFFFFFFF vs FSSSFSSS, indexer
  64 x 128, k=2048, attention 16 / 1 x 128, correlated layers.
* ``decode_32k``    B=32 sequences, one new query each over a 32768-token
  cache (q_offset = 32767), 16 layers (FSSS)x4, indexer 64 x 128, k=2048.
* ``sweep_<L>``     B=1, one layer, L in {4096, 16384, 65536, 131072},
  indexer 64 x 128, k=2048.
* ``layer_32k``     B=1, one F layer at L=32768 with the sweep's shapes (the
  smallest prefill whose late rows gather K/V rows; used for kernel profiles).

Correlated layers: the pages report that adjacent layers share 70-100% of
their top-k selections (IndexCache technical summary, Probleemstelling; kualia
review, "The Redundancy That Was Sitting There").  Synthetic layers get that
property from a shared component: for an indexer tensor X of layer l,
X_l = sqrt(rho) * X_shared + sqrt(1 - rho) * E_l, where the shared key part is
low rank (rank 16, rescaled to unit variance) and E_l is fresh noise.  K and V
mix a shared low-rank part with rho_kv = 0.5; attention queries are drawn
independently per layer.  Every tensor is finally divided by sqrt(last dim).
Seeds: tiny_prefill uses one generator seeded 0; the others seed each tensor
with 1000*cfg + 10*layer + tensor_id (shared parts use layer 99).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch

RANK = 16
RHO_KV = 0.5
# rho for the indexer tensors; chosen by measuring the adjacent-layer top-k
# overlap of prefill_8k with the oracle (it lands inside the 70-100% band).
RHO_INDEXER = 0.98

_TID = {"q_idx": 0, "k_idx": 1, "w": 2, "q": 3, "k": 4, "v": 5,
        "a": 6, "p_idx": 7, "p_k": 8, "p_v": 9}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Lq: int
    Lk: int
    n_layers: int
    H_I: int
    d_I: int
    k: int
    Hq: int
    d: int
    pattern: str
    q_offset: int = 0
    cfg_id: int = 0
    correlated: bool = True

    @property
    def dims(self) -> Dict[str, int]:
        return dict(B=self.B, Lq=self.Lq, Lk=self.Lk, q_offset=self.q_offset, H_I=self.H_I,
                    d_I=self.d_I, Hq=self.Hq, Hkv=1, d=self.d, k=self.k)


def _prefill(name, L, n_layers, H_I, d_I, k, Hq, d, pattern, cfg_id, correlated=True):
    return Workload(name, 1, L, L, n_layers, H_I, d_I, k, Hq, d, pattern, 0, cfg_id, correlated)


WORKLOADS: Dict[str, Workload] = {
    "tiny_prefill": _prefill("tiny_prefill", 512, 4, 4, 64, 64, 8, 64, "FSSS", 1, False),
    "prefill_8k": _prefill("prefill_8k", 8192, 8, 32, 128, 2048, 16, 128, "FSSSFSSS", 2),
    "prefill_64k": _prefill("prefill_64k", 65536, 8, 64, 128, 2048, 16, 128, "FSSSFSSS", 3),
    "decode_32k": Workload("decode_32k", 32, 1, 32768, 16, 64, 128, 2048, 16, 128, "FSSS" * 4,
                           32767, 4, True),
}
for _L in (4096, 16384, 65536, 131072):
    WORKLOADS[f"sweep_{_L // 1024}k"] = _prefill(f"sweep_{_L // 1024}k", _L, 1, 64, 128, 2048, 16,
                                                 128, "F", 5)
# A single F layer at L=32768 (shapes of the sweep), long enough that most of
# its rows gather their K/V rows (t >= 6k = 12288), for kernel profiles.
WORKLOADS["layer_32k"] = _prefill("layer_32k", 32768, 1, 64, 128, 2048, 16, 128, "F", 6)


def custom(name: str = "custom", *, B=1, Lq, Lk=None, n_layers=1, H_I=4, d_I=64, k=64, Hq=8,
           d=64, pattern=None, q_offset=0, cfg_id=9, correlated=False) -> Workload:
    """A workload of arbitrary shape (tests use it for ragged and edge sizes)."""
    Lk = Lq + q_offset if Lk is None else Lk
    pattern = pattern or ("F" + "S" * (n_layers - 1))
    return Workload(name, B, Lq, Lk, n_layers, H_I, d_I, k, Hq, d, pattern, q_offset, cfg_id,
                    correlated)


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, seed: int, device="cpu") -> torch.Tensor:
    return torch.randn(*shape, generator=_gen(seed, device), dtype=torch.float32, device=device)


def _seed(wl: Workload, layer: int, name: str) -> int:
    return 1000 * wl.cfg_id + 10 * layer + _TID[name]


def _low_rank(rows: int, cols: int, wl: Workload, pname: str, batch: int,
              device="cpu") -> torch.Tensor:
    """Unit-variance rank-16 matrix [batch, rows, cols] shared by every layer."""
    a = _randn((batch, rows, RANK), _seed(wl, 99, "a"), device)
    p = _randn((RANK, cols), _seed(wl, 99, pname), device)
    return (a @ p) / math.sqrt(RANK)


def _mix(shared: torch.Tensor, noise: torch.Tensor, rho: float) -> torch.Tensor:
    return math.sqrt(rho) * shared + math.sqrt(1.0 - rho) * noise


def make_layers(wl: Workload, layers: Optional[List[int]] = None, indexer_for_all: bool = True,
                rho: float = RHO_INDEXER, device="cpu") -> List[Dict[str, torch.Tensor]]:
    """Draw the per-layer inputs (bf16 operands, fp32 head weights).

    Returns a list of dicts with 'q', 'k', 'v' ([B,L,Hq,d] and [B,Lk,1,d]) and,
    for F layers (or every layer when indexer_for_all), 'q_idx' [B,Lq,H_I,d_I],
    'k_idx' [B,Lk,d_I], 'w' [B,Lq,H_I].  device='cuda' draws with device
    generators (same seeds, different random streams than the CPU ones) for
    workloads too large to draw on the host.
    """
    B, Lq, Lk = wl.B, wl.Lq, wl.Lk
    layers = list(range(wl.n_layers)) if layers is None else list(layers)
    out: List[Dict[str, torch.Tensor]] = []
    if not wl.correlated:
        # One generator seeded 0 (or cfg_id*1000) draws every tensor in a fixed order.
        g = _gen(0 if wl.cfg_id == 1 else 1000 * wl.cfg_id)
        per_layer = []
        for l in range(wl.n_layers):
            t = {}
            t["q_idx"] = torch.randn(B, Lq, wl.H_I, wl.d_I, generator=g) / math.sqrt(wl.d_I)
            t["k_idx"] = torch.randn(B, Lk, wl.d_I, generator=g) / math.sqrt(wl.d_I)
            t["w"] = torch.randn(B, Lq, wl.H_I, generator=g) / math.sqrt(wl.H_I)
            t["q"] = torch.randn(B, Lq, wl.Hq, wl.d, generator=g) / math.sqrt(wl.d)
            t["k"] = torch.randn(B, Lk, 1, wl.d, generator=g) / math.sqrt(wl.d)
            t["v"] = torch.randn(B, Lk, 1, wl.d, generator=g) / math.sqrt(wl.d)
            per_layer.append(t)
        for l in layers:
            t = per_layer[l]
            d = {n: t[n].to(torch.bfloat16) for n in ("q", "k", "v")}
            if indexer_for_all or wl.pattern[l] in "F1":
                d["q_idx"] = t["q_idx"].to(torch.bfloat16)
                d["k_idx"] = t["k_idx"].to(torch.bfloat16)
                d["w"] = t["w"].contiguous()
            # drawn on the host (the fixed-order stream), then placed on `device`
            out.append({n: v.to(device) for n, v in d.items()})
        return out

    dev = device
    k_shared = _low_rank(Lk, wl.d_I, wl, "p_idx", B, dev)
    kv_k = _low_rank(Lk, wl.d, wl, "p_k", B, dev)
    kv_v = _low_rank(Lk, wl.d, wl, "p_v", B, dev)
    q_shared = w_shared = None
    for l in layers:
        d: Dict[str, torch.Tensor] = {}
        d["q"] = (_randn((B, Lq, wl.Hq, wl.d), _seed(wl, l, "q"), dev) / math.sqrt(wl.d)).to(torch.bfloat16)
        ek = _randn((B, Lk, wl.d), _seed(wl, l, "k"), dev)
        ev = _randn((B, Lk, wl.d), _seed(wl, l, "v"), dev)
        d["k"] = (_mix(kv_k, ek, RHO_KV) / math.sqrt(wl.d)).to(torch.bfloat16).reshape(B, Lk, 1, wl.d)
        d["v"] = (_mix(kv_v, ev, RHO_KV) / math.sqrt(wl.d)).to(torch.bfloat16).reshape(B, Lk, 1, wl.d)
        if indexer_for_all or wl.pattern[l] in "F1":
            if q_shared is None:
                q_shared = _randn((B, Lq, wl.H_I, wl.d_I), _seed(wl, 99, "q_idx"), dev)
                w_shared = _randn((B, Lq, wl.H_I), _seed(wl, 99, "w"), dev)
            qi = _mix(q_shared, _randn((B, Lq, wl.H_I, wl.d_I), _seed(wl, l, "q_idx"), dev), rho)
            ki = _mix(k_shared, _randn((B, Lk, wl.d_I), _seed(wl, l, "k_idx"), dev), rho)
            wi = _mix(w_shared, _randn((B, Lq, wl.H_I), _seed(wl, l, "w"), dev), rho)
            d["q_idx"] = (qi / math.sqrt(wl.d_I)).to(torch.bfloat16)
            d["k_idx"] = (ki / math.sqrt(wl.d_I)).to(torch.bfloat16)
            d["w"] = (wi / math.sqrt(wl.H_I)).contiguous()
        out.append(d)
    return out


def sample_rows(wl: Workload, n: int = 256, seed: int = 7) -> List[int]:
    """A bounded, deterministic sample of flattened query rows b*Lq + i.

    It always holds the first and last row of each sequence and the rows
    around position k-1 (where rows stop selecting every visible position);
    the rest is spread evenly over the remaining rows.
    """
    total = wl.B * wl.Lq
    if total <= n:
        return list(range(total))
    want = set()
    for b in range(wl.B):
        base = b * wl.Lq
        want.update({base, base + wl.Lq - 1})
        for t in (wl.k - 2, wl.k - 1, wl.k, wl.k + 1):
            i = t - wl.q_offset
            if 0 <= i < wl.Lq:
                want.add(base + i)
    g = _gen(seed)
    rest = n - len(want)
    if rest > 0:
        strata = torch.linspace(0, total, rest + 1)
        for a, b in zip(strata[:-1].tolist(), strata[1:].tolist()):
            lo, hi = int(a), max(int(a) + 1, int(b))
            want.add(int(torch.randint(lo, hi, (1,), generator=g).item()))
    return sorted(want)[:max(n, len(want))]
