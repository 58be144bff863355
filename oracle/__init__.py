"""CPU oracle for the IndexCache sparse-attention layer stack.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (the CUDA library and its binding) never imports,
links or runs anything here, and nothing here imports the product.

The arithmetic lives in ``oracle.c`` (plain C, fp64 accumulation, OpenMP over
query rows).  This module builds it with gcc, marshals numpy / torch-CPU arrays
into it, and runs the layer loop of the IndexCache inference path:

* "IndexCache: Accelerating Sparse Attention via Cross-Layer Index Reuse"
  (skill page, Step 3, ``IndexCacheManager.get_indices_for_layer``): an F layer
  computes fresh indices and stores them as the cached indices; an S layer
  returns the cached indices and fails when none exist yet.
* Same paper (Dutch technical summary, Methodologie): S layers inherit the
  top-k indices of the nearest preceding F layer.
* kualia.ai review ("The Redundancy That Was Sitting There"): the cache is
  one scratch tensor of indices that each F layer replaces.

Pattern characters: 'F' or '1' = full layer, 'S' or '0' = shared layer (the
skill page's code uses '1'/'0', the prose uses F/S).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None
# Host threads (a row-per-core pool) may ask for the library at the same time:
# one of them builds and loads it, the others wait.
_lock = threading.RLock()


class NoCachedIndices(ValueError):
    """An S layer ran before any F layer filled the index cache."""


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            # a name of this process and thread: concurrent builds (several
            # processes) each replace the library atomically with a whole file
            tmp = f"{_LIB}.{os.getpid()}.{threading.get_ident()}.tmp"
            cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall",
                   "-o", tmp, _SRC, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        build()
        lib = ctypes.CDLL(_LIB)
        P, I, L, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.or_indexer_scores.argtypes = [P, P, P, I, I, I, I, I, I, P, L, P]
        lib.or_topk_sort.argtypes = [P, P, L, I, I, P]
        lib.or_topk_count.argtypes = [P, P, L, I, I, P]
        lib.or_sparse_attn.argtypes = [P, P, P, P, I, I, I, I, I, I, I, D, P, L, P, P]
        lib.or_dense_attn.argtypes = [P, P, P, I, I, I, I, I, I, D, P, L, P, P]
        lib.or_index_overlap.argtypes = [P, P, L, I, I, P]
        for f in ("or_indexer_scores", "or_topk_sort", "or_topk_count", "or_sparse_attn",
                  "or_dense_attn", "or_num_threads", "or_index_overlap"):
            getattr(lib, f).restype = ctypes.c_int
        lib.or_set_num_threads.argtypes = [I]
        lib.or_set_num_threads.restype = None
        _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(_load().or_num_threads())


def set_num_threads(n: int) -> None:
    """Threads this host thread's later oracle calls use."""
    _load().or_set_num_threads(int(n))


# ---------------------------------------------------------------- marshalling

def _bf16_bits(x) -> np.ndarray:
    """bf16 payload as a contiguous uint16 array (torch bf16 tensor or uint16 array)."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("bf16 operands are passed as uint16 bit patterns")
        return np.ascontiguousarray(x)
    import torch  # only for unpacking a torch tensor handed in by a test
    if x.dtype != torch.bfloat16:
        raise TypeError("expected a bfloat16 tensor")
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _f32(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.float32)
    return x.detach().cpu().contiguous().float().numpy()


def _i32(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.int32)
    return x.detach().cpu().contiguous().numpy().astype(np.int32)


def _rows(rows, total):
    if rows is None:
        return None, total
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    return r, int(r.shape[0])


def _ptr(a) -> Optional[int]:
    return None if a is None else a.ctypes.data


# ---------------------------------------------------------------- steps

def indexer_scores(q_idx, k_idx, w, q_offset: int = 0, rows=None) -> np.ndarray:
    """Lightning indexer scores in fp64 for the requested flattened rows.

    q_idx [B,Lq,H,dI] bf16, k_idx [B,Lk,dI] bf16, w [B,Lq,H] fp32 ->
    [n_rows, Lk] float64 with -inf at invisible positions (s > t).
    """
    qb, kb, wf = _bf16_bits(q_idx), _bf16_bits(k_idx), _f32(w)
    B, Lq, H, dI = qb.shape
    Lk = kb.shape[1]
    if kb.shape != (B, Lk, dI) or wf.shape != (B, Lq, H):
        raise ValueError("shape mismatch")
    r, n = _rows(rows, B * Lq)
    out = np.empty((n, Lk), dtype=np.float64)
    rc = _load().or_indexer_scores(_ptr(qb), _ptr(kb), _ptr(wf), B, Lq, Lk, H, dI, q_offset,
                                   _ptr(r), n, _ptr(out))
    if rc:
        raise ValueError(f"or_indexer_scores failed ({rc})")
    return out


def row_positions(B: int, Lq: int, q_offset: int, rows=None) -> np.ndarray:
    """Absolute position t of each requested flattened row."""
    r = np.arange(B * Lq, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    return (r % Lq) + q_offset


def topk_sort(scores, tpos, k: int) -> np.ndarray:
    """Sort-based top-k of float32 score rows -> int32 [n_rows, k] (ascending, -1 padded)."""
    s = _f32(scores)
    n, Lk = s.shape
    tp = np.ascontiguousarray(np.asarray(tpos, dtype=np.int64))
    idx = np.empty((n, k), dtype=np.int32)
    rc = _load().or_topk_sort(_ptr(s), _ptr(tp), n, Lk, k, _ptr(idx))
    if rc:
        raise ValueError(f"or_topk_sort failed ({rc})")
    return idx


def topk_count(scores, tpos, k: int) -> np.ndarray:
    """Brute-force count form of the same top-k (tiny rows only, O(n^2) per row)."""
    s = _f32(scores)
    n, Lk = s.shape
    tp = np.ascontiguousarray(np.asarray(tpos, dtype=np.int64))
    idx = np.empty((n, k), dtype=np.int32)
    rc = _load().or_topk_count(_ptr(s), _ptr(tp), n, Lk, k, _ptr(idx))
    if rc:
        raise ValueError(f"or_topk_count failed ({rc})")
    return idx


def _attn_shapes(q, K, V):
    qb, Kb, Vb = _bf16_bits(q), _bf16_bits(K), _bf16_bits(V)
    B, Lq, Hq, d = qb.shape
    Lk = Kb.shape[1]
    Kb = Kb.reshape(B, Lk, -1)
    Vb = Vb.reshape(B, Lk, -1)
    if Kb.shape[2] != d or Vb.shape != Kb.shape:
        raise ValueError("K/V must be [B, Lk, 1, d] or [B, Lk, d] with one KV head")
    return qb, Kb, Vb, B, Lq, Lk, Hq, d


def sparse_attn(q, K, V, idx_rows, q_offset: int = 0, scale: float = 0.0, rows=None):
    """Softmax attention over the cached positions, fp64.

    idx_rows holds one index row per requested row ([n_rows, k] int32, -1 =
    empty).  Returns (out [n_rows, Hq, d] float64, lse [n_rows, Hq] float64).
    """
    qb, Kb, Vb, B, Lq, Lk, Hq, d = _attn_shapes(q, K, V)
    ix = _i32(idx_rows)
    r, n = _rows(rows, B * Lq)
    ix = ix.reshape(n, -1)
    k = ix.shape[1]
    out = np.empty((n, Hq, d), dtype=np.float64)
    lse = np.empty((n, Hq), dtype=np.float64)
    rc = _load().or_sparse_attn(_ptr(qb), _ptr(Kb), _ptr(Vb), _ptr(ix), B, Lq, Lk, Hq, d, k,
                                q_offset, float(scale), _ptr(r), n, _ptr(out), _ptr(lse))
    if rc:
        raise ValueError(f"or_sparse_attn failed ({rc})")
    return out, lse


def dense_attn(q, K, V, q_offset: int = 0, scale: float = 0.0, rows=None):
    """Causal softmax attention over every visible position s <= t, fp64."""
    qb, Kb, Vb, B, Lq, Lk, Hq, d = _attn_shapes(q, K, V)
    r, n = _rows(rows, B * Lq)
    out = np.empty((n, Hq, d), dtype=np.float64)
    lse = np.empty((n, Hq), dtype=np.float64)
    rc = _load().or_dense_attn(_ptr(qb), _ptr(Kb), _ptr(Vb), B, Lq, Lk, Hq, d, q_offset,
                               float(scale), _ptr(r), n, _ptr(out), _ptr(lse))
    if rc:
        raise ValueError(f"or_dense_attn failed ({rc})")
    return out, lse


def index_overlap(idx_a, idx_b, Lk: int) -> np.ndarray:
    """Per row of two index tensors ([n_rows, k] int32, -1 = empty), the set
    sizes (|A & B|, |A|, |B|) as int32 [n_rows, 3] (skill page, Step 1)."""
    a, b = _i32(idx_a), _i32(idx_b)
    if a.shape != b.shape:
        raise ValueError("index tensors differ in shape")
    k = a.shape[-1]
    a = a.reshape(-1, k)
    b = b.reshape(-1, k)
    out = np.empty((a.shape[0], 3), dtype=np.int32)
    rc = _load().or_index_overlap(_ptr(a), _ptr(b), a.shape[0], k, int(Lk), _ptr(out))
    if rc:
        raise ValueError(f"or_index_overlap failed ({rc})")
    return out


def overlap_fraction(counts, k: int) -> np.ndarray:
    """|A & B| / k per row: the share of a layer's k selections another layer
    also selects (kualia.ai review: adjacent layers share 70-100%)."""
    return np.asarray(counts)[:, 0] / float(k)


def jaccard(counts) -> np.ndarray:
    """|A & B| / (|A | B| + 1e-8) per row (skill page, Step 1)."""
    c = np.asarray(counts, dtype=np.float64)
    return c[:, 0] / (c[:, 1] + c[:, 2] - c[:, 0] + 1e-8)


def is_full(c: str) -> bool:
    if c in ("F", "1"):
        return True
    if c in ("S", "0"):
        return False
    raise ValueError(f"pattern character {c!r} is neither F/1 nor S/0")


def layer_stack(pattern: str, layers: Sequence[dict], k: int, q_offset: int = 0,
                scale: float = 0.0, rows=None):
    """Run the F/S layer loop over the requested rows.

    layers[l] holds 'q', 'k', 'v' and, for F layers, 'q_idx', 'k_idx', 'w'.
    Returns (outs, idxs, lses): per layer the fp64 attention output, the int32
    index rows that layer attended over, and the fp64 log-sum-exp.
    """
    if len(pattern) != len(layers):
        raise ValueError("pattern length must equal the number of layers")
    cached = None
    outs, idxs, lses = [], [], []
    for l, c in enumerate(pattern):
        L = layers[l]
        if is_full(c):
            qi = _bf16_bits(L["q_idx"])
            B, Lq = qi.shape[0], qi.shape[1]
            sc = indexer_scores(qi, L["k_idx"], L["w"], q_offset, rows)
            cached = topk_sort(sc.astype(np.float32), row_positions(B, Lq, q_offset, rows), k)
        elif cached is None:
            raise NoCachedIndices(f"layer {l} is shared, but no full layer before it has "
                                  "filled the index cache")
        o, lse = sparse_attn(L["q"], L["k"], L["v"], cached, q_offset, scale, rows)
        outs.append(o)
        idxs.append(cached)
        lses.append(lse)
    return outs, idxs, lses
