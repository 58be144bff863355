"""Sharding the layer stack over GPUs (one process per GPU, no data-path exchange).

Query rows are independent given the prefix: row t of a layer needs only
q / q_I / w of row t and K, V, k_I of positions <= t, and the index cache of
row t is written and read by row t alone (IndexCache: an F layer's indexer
scores every preceding token of each query and keeps its top-k; the S layers
after it reuse that row's k positions).  So a stack splits over ranks by rows
with no collective on the data path:

* one long sequence (B = 1, prefill): zig-zag row chunks.  The rows are cut
  into 2 x world equal contiguous chunks and rank r takes chunks r and
  2*world-1-r, pairing cheap early rows with expensive late ones under the
  causal mask.  Every chunk is an ordinary stack call over rows
  [i0, i0 + n) of the sequence with q_offset + i0 and the full K/V/k_I prefix.
* a batch (B > 1, decode or many prompts): whole sequences, B / world each.

Each rank keeps its own outputs; gathering them (an all-gather per layer) is
the caller's choice and not part of the path.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence, Tuple


@dataclass(frozen=True)
class RowChunk:
    b0: int          # first sequence
    nb: int          # sequences
    i0: int          # first query row of each sequence (relative to q_offset)
    n: int           # query rows


def row_cost(t: int) -> float:
    """Relative cost of query row t: the indexer and the top-k scale with the
    t + 1 visible positions, and they dominate long prefills."""
    return float(t + 1)


def zigzag_chunks(Lq: int, world: int, rank: int, align: int = 128) -> List[Tuple[int, int]]:
    """Rank `rank`'s row chunks (i0, n) of one sequence of Lq rows.

    Chunk boundaries are multiples of `align` rows (so every chunk starts on
    a whole query block of the kernels) except at Lq; empty chunks are
    dropped.  Over all ranks the chunks cover [0, Lq) exactly once.
    """
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    m = 2 * world
    bounds = [min(Lq, (round(Lq * c / m) + align - 1) // align * align) for c in range(m + 1)]
    bounds[0], bounds[-1] = 0, Lq
    out = []
    for c in (rank, m - 1 - rank):
        i0, i1 = bounds[c], bounds[c + 1]
        if i1 > i0:
            out.append((i0, i1 - i0))
    return out


def shard(B: int, Lq: int, world: int, rank: int, align: int = 128) -> List[RowChunk]:
    """The work of rank `rank` as RowChunks: zig-zag rows when B == 1, whole
    sequences otherwise (the first B % world ranks take one more)."""
    if B == 1:
        return [RowChunk(0, 1, i0, n) for i0, n in zigzag_chunks(Lq, world, rank, align)]
    base, extra = divmod(B, world)
    nb = base + (1 if rank < extra else 0)
    b0 = rank * base + min(rank, extra)
    return [RowChunk(b0, nb, 0, Lq)] if nb > 0 else []


def chunk_cost(ch: RowChunk, q_offset: int) -> float:
    return ch.nb * sum(row_cost(q_offset + ch.i0 + i) for i in range(ch.n))


def slice_layers(layers: Sequence[dict], ch: RowChunk) -> List[dict]:
    """Per layer, the chunk's view of its inputs: rows [i0, i0+n) of q, q_idx
    and w for sequences [b0, b0+nb); K, V and k_I keep every position."""
    out = []
    for L in layers:
        d = {}
        for name, t in L.items():
            t = t[ch.b0: ch.b0 + ch.nb]
            if name in ("q", "q_idx", "w"):
                t = t[:, ch.i0: ch.i0 + ch.n]
            d[name] = t.contiguous()
        out.append(d)
    return out


class ShardedStack:
    """A rank's share of a layer stack: one LayerStack per row chunk, all on
    this process's GPU and stream.  outs[c][l] is chunk c's output of layer l
    ([nb, n, Hq, d]); chunks[c] says which rows they are."""

    def __init__(self, pattern: str, layers: Sequence[dict], dims_full, world: int, rank: int,
                 align: int = 128, **stack_kw):
        from . import indexcache as ic
        d = dims_full
        self.chunks = shard(d.B, d.Lq, world, rank, align)
        self.stacks = []
        for ch in self.chunks:
            dims = ic.make_dims(ch.nb, ch.n, d.Lk, d.q_offset + ch.i0, d.H_I, d.d_I, d.Hq, d.d,
                                d.k, d.scale, d.Hkv)
            self.stacks.append(ic.LayerStack(pattern, slice_layers(layers, ch), dims, **stack_kw))

    def forward(self, stream=None):
        for st in self.stacks:
            st.forward(stream)
        return [st.outs for st in self.stacks]
