"""ctypes binding of libindexcache.so (argument marshalling only).

Every function here takes torch CUDA tensors, checks dtype/shape/contiguity,
and passes raw device pointers to the C ABI of the same name
(include/indexcache.h).  No step of the computation happens in Python, and
there is no fallback: importing this module fails loudly when the CUDA
library has not been built, and each call raises IndexCacheError on a
non-zero status.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libindexcache.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m lightning_indexer_top_relu_b200.build` "
        "(there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

IC_OK = 0
STATUS = {0: "IC_OK", 1: "IC_ERR_INVALID_ARG", 2: "IC_ERR_UNSUPPORTED",
          3: "IC_ERR_NO_CACHED_INDICES", 4: "IC_ERR_WORKSPACE_TOO_SMALL", 5: "IC_ERR_CUDA",
          6: "IC_ERR_TIMEOUT"}
EXPORTS = ("ic_status_string", "ic_last_error_message", "ic_get_last_device_error",
           "ic_indexer_scores", "ic_topk_select", "ic_sparse_attn",
           "ic_sparse_attn_workspace_bytes", "ic_layer_stack_workspace_bytes",
           "ic_layer_stack_forward", "ic_layer_stack_forward_events", "ic_selftest_wait_timeout",
           "ic_sparse_attn_no_alloc", "ic_kernel_launch_count", "ic_sparse_attn_unique",
           "ic_sparse_attn_unique_workspace_bytes", "ic_index_overlap",
           "ic_layer_stack_dense_rows", "ic_layer_stack_forward_opts",
           "ic_layer_stack_fused_fallback_blocks")

MARKS_PER_LAYER = 5        # IC_MARKS_PER_LAYER


class IndexCacheError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.ic_last_error_message().decode(errors="replace")
        super().__init__(f"{where}: {STATUS.get(status, status)}: {msg}")


class NoCachedIndices(IndexCacheError, ValueError):
    """A shared layer came before any full layer (IC_ERR_NO_CACHED_INDICES).
    Also a ValueError: the failure a caller of a Python index-cache lookup
    expects when no indices have been stored yet."""


class ICLayer(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("q_idx", ctypes.c_void_p), ("k_idx", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("idx_dump", ctypes.c_void_p)]


class ICStackOptions(ctypes.Structure):
    """ic_stack_options: fused_topk -1 (library's choice), 0 (store the scores,
    then top-k) or 1 (fused indexer -> top-k); z the threshold margin."""
    _fields_ = [("fused_topk", ctypes.c_int), ("z", ctypes.c_float)]


class ICDims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Lq", ctypes.c_int), ("Lk", ctypes.c_int),
                ("q_offset", ctypes.c_int), ("H_I", ctypes.c_int), ("d_I", ctypes.c_int),
                ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
                ("k", ctypes.c_int), ("scale", ctypes.c_float)]


_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_lib.ic_status_string.restype = ctypes.c_char_p
_lib.ic_status_string.argtypes = [_I]
_lib.ic_last_error_message.restype = ctypes.c_char_p
_lib.ic_last_error_message.argtypes = []
_lib.ic_get_last_device_error.restype = _I
_lib.ic_get_last_device_error.argtypes = [_P]
_lib.ic_indexer_scores.restype = _I
_lib.ic_indexer_scores.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P]
_lib.ic_topk_select.restype = _I
_lib.ic_topk_select.argtypes = [_P, _I, _I, _I, _I, _I, _P, _P]
_lib.ic_sparse_attn.restype = _I
_lib.ic_sparse_attn.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P,
                                _Z, _P]
_lib.ic_sparse_attn_no_alloc.restype = _I
_lib.ic_sparse_attn_no_alloc.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P,
                                         _P, _P]
_lib.ic_sparse_attn_unique.restype = _I
_lib.ic_sparse_attn_unique.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P,
                                       _P, _Z, _P]
_lib.ic_sparse_attn_unique_workspace_bytes.restype = _Z
_lib.ic_sparse_attn_unique_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I, _I]
_lib.ic_sparse_attn_workspace_bytes.restype = _Z
_lib.ic_sparse_attn_workspace_bytes.argtypes = [_I, _I, _I, _I, _I]
_lib.ic_layer_stack_dense_rows.restype = _I
_lib.ic_layer_stack_dense_rows.argtypes = [ctypes.POINTER(ICDims), _Z]
_lib.ic_layer_stack_workspace_bytes.restype = _Z
_lib.ic_layer_stack_workspace_bytes.argtypes = [ctypes.POINTER(ICDims), _I, ctypes.c_longlong]
_lib.ic_selftest_wait_timeout.restype = _I
_lib.ic_selftest_wait_timeout.argtypes = [_I, _P]
_lib.ic_layer_stack_forward_events.restype = _I
_lib.ic_layer_stack_forward_events.argtypes = [ctypes.c_char_p, _I, ctypes.POINTER(ICLayer),
                                               ctypes.POINTER(ICDims), _P, _P, _Z, _P, _P]
_lib.ic_index_overlap.restype = _I
_lib.ic_index_overlap.argtypes = [_P, _P, ctypes.c_longlong, _I, _I, _P, _P]
_lib.ic_kernel_launch_count.restype = ctypes.c_ulonglong
_lib.ic_kernel_launch_count.argtypes = []
_lib.ic_layer_stack_forward_opts.restype = _I
_lib.ic_layer_stack_forward_opts.argtypes = [ctypes.c_char_p, _I, ctypes.POINTER(ICLayer),
                                             ctypes.POINTER(ICDims), ctypes.POINTER(ICStackOptions),
                                             _P, _P, _Z, _P, _P]
_lib.ic_layer_stack_fused_fallback_blocks.restype = _I
_lib.ic_layer_stack_fused_fallback_blocks.argtypes = [ctypes.POINTER(ICDims),
                                                      ctypes.POINTER(ICStackOptions), _P, _Z, _P,
                                                      ctypes.POINTER(ctypes.c_int)]
_lib.ic_layer_stack_forward.restype = _I
_lib.ic_layer_stack_forward.argtypes = [ctypes.c_char_p, _I, ctypes.POINTER(ICLayer),
                                        ctypes.POINTER(ICDims), _P, _P, _Z, _P]


def lib() -> ctypes.CDLL:
    return _lib


def _check(rc: int, where: str):
    if rc != IC_OK:
        if rc == 3:
            raise NoCachedIndices(rc, where)
        raise IndexCacheError(rc, where)


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor") -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        # the library launches on the current device and would dereference
        # another GPU's memory
        raise ValueError(f"{name} is on {t.device}, but the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _expect(t: Optional[torch.Tensor], shape, name: str) -> None:
    """A caller tensor must have exactly the shape the call derives from its
    leading operand: the C layer sees only pointers and sizes, so a smaller
    tensor would let a kernel read or write past its end."""
    if t is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _dims_of(t: torch.Tensor, n: int, name: str):
    if t.dim() != n:
        raise ValueError(f"{name} must have {n} dimensions, got shape {tuple(t.shape)}")
    return tuple(t.shape)


def _kv_shapes(q, k, v):
    """(B, Lq, Hq, d, Lk, Hkv) of an attention call: q [B,Lq,Hq,d]; k and v
    [B,Lk,Hkv,d] or [B,Lk,d] (one KV head), both the same."""
    B, Lq, Hq, d = _dims_of(q, 4, "q")
    if k.dim() == 4:
        Lk, Hkv = k.shape[1], k.shape[2]
        _expect(k, (B, Lk, Hkv, d), "k")
    else:
        Lk, Hkv = _dims_of(k, 3, "k")[1], 1
        _expect(k, (B, Lk, d), "k")
    _expect(v, tuple(k.shape), "v")
    return B, Lq, Hq, d, Lk, Hkv


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def get_last_device_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error status."""
    return int(_lib.ic_get_last_device_error(_stream(stream)))


def index_overlap(idx_a, idx_b, Lk: int, counts=None, stream=None):
    """Per-row (|A & B|, |A|, |B|) of two [..., k] int32 index tensors on the
    device, as int32 [n_rows, 3] (ic_index_overlap)."""
    if idx_a.shape != idx_b.shape:
        raise ValueError("index tensors differ in shape")
    k = idx_a.shape[-1]
    n_rows = idx_a.numel() // k
    if counts is None:
        counts = torch.empty(n_rows, 3, device=idx_a.device, dtype=torch.int32)
    _expect(counts, (n_rows, 3), "counts")
    rc = _lib.ic_index_overlap(_ptr(idx_a, torch.int32, "idx_a"), _ptr(idx_b, torch.int32, "idx_b"),
                               n_rows, k, int(Lk), _ptr(counts, torch.int32, "counts"),
                               _stream(stream))
    _check(rc, "ic_index_overlap")
    return counts


def kernel_launch_count() -> int:
    """Kernel launches the library has issued in this process so far."""
    return int(_lib.ic_kernel_launch_count())


def selftest_wait_timeout(timeout_us: int = 20000, stream=None) -> None:
    """Launches the bounded-wait self test (see include/indexcache.h)."""
    _check(_lib.ic_selftest_wait_timeout(int(timeout_us), _stream(stream)), "ic_selftest_wait_timeout")


def indexer_scores(q_idx, k_idx, w, q_offset: int = 0, out=None, stream=None) -> torch.Tensor:
    """scores [B,Lq,Lk] fp32 from q_idx [B,Lq,H_I,d_I] bf16, k_idx [B,Lk,d_I] bf16, w [B,Lq,H_I] fp32."""
    B, Lq, H, dI = _dims_of(q_idx, 4, "q_idx")
    Lk = _dims_of(k_idx, 3, "k_idx")[1]
    _expect(k_idx, (B, Lk, dI), "k_idx")
    _expect(w, (B, Lq, H), "w")
    if out is None:
        out = torch.empty(B, Lq, Lk, device=q_idx.device, dtype=torch.float32)
    _expect(out, (B, Lq, Lk), "out")
    rc = _lib.ic_indexer_scores(_ptr(q_idx, torch.bfloat16, "q_idx"), _ptr(k_idx, torch.bfloat16, "k_idx"),
                                _ptr(w, torch.float32, "w"), B, Lq, Lk, H, dI, q_offset,
                                _ptr(out, torch.float32, "scores"), _stream(stream))
    _check(rc, "ic_indexer_scores")
    return out


def topk_select(scores, k: int, q_offset: int = 0, out=None, stream=None) -> torch.Tensor:
    """idx [B,Lq,k] int32 (ascending positions, -1 padded) from scores [B,Lq,Lk] fp32."""
    B, Lq, Lk = _dims_of(scores, 3, "scores")
    if out is None:
        out = torch.empty(B, Lq, k, device=scores.device, dtype=torch.int32)
    _expect(out, (B, Lq, k), "out")
    rc = _lib.ic_topk_select(_ptr(scores, torch.float32, "scores"), B, Lq, Lk, q_offset, k,
                             _ptr(out, torch.int32, "idx"), _stream(stream))
    _check(rc, "ic_topk_select")
    return out


def sparse_attn_workspace_bytes(B: int, Lq: int, Hq: int, d: int, k: int) -> int:
    return int(_lib.ic_sparse_attn_workspace_bytes(B, Lq, Hq, d, k))


def sparse_attn(q, k, v, idx, q_offset: int = 0, scale: float = 0.0, out=None, lse=None,
                want_lse: bool = True, ws=None, stream=None):
    """(out [B,Lq,Hq,d] bf16, lse [B,Lq,Hq] fp32) over the positions in idx [B,Lq,k] int32."""
    B, Lq, Hq, d, Lk, Hkv = _kv_shapes(q, k, v)
    kslots = _dims_of(idx, 3, "idx")[2]
    _expect(idx, (B, Lq, kslots), "idx")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, Lq, Hq, device=q.device, dtype=torch.float32)
    _expect(out, (B, Lq, Hq, d), "out")
    _expect(lse, (B, Lq, Hq), "lse")
    if ws is None:
        nbytes = sparse_attn_workspace_bytes(B, Lq, Hq, d, kslots)
        ws = torch.empty(max(nbytes, 1), device=q.device, dtype=torch.uint8) if nbytes else None
    rc = _lib.ic_sparse_attn(_ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                             _ptr(v, torch.bfloat16, "v"), _ptr(idx, torch.int32, "idx"), B, Lq,
                             Lk, Hq, Hkv, d, kslots, q_offset, float(scale),
                             _ptr(out, torch.bfloat16, "out"), _ptr(lse, torch.float32, "lse"),
                             _ptr(ws, None, "ws"), 0 if ws is None else ws.numel() * ws.element_size(),
                             _stream(stream))
    _check(rc, "ic_sparse_attn")
    return out, lse


def sparse_attn_unique_workspace_bytes(B: int, Lq: int, Lk: int, q_offset: int, Hq: int, d: int,
                                       k: int) -> int:
    return int(_lib.ic_sparse_attn_unique_workspace_bytes(B, Lq, Lk, q_offset, Hq, d, k))


def sparse_attn_unique(q, k, v, idx, q_offset: int = 0, scale: float = 0.0, out=None, lse=None,
                       want_lse: bool = True, ws=None, stream=None):
    """ic_sparse_attn_unique: the layer stack's attention step for index rows
    that hold each position at most once (dense-masked rows t < 6k when the
    workspace allows, gathered rows otherwise).  ws=None allocates the full
    workspace; pass an empty tensor to force the gather path."""
    B, Lq, Hq, d, Lk, Hkv = _kv_shapes(q, k, v)
    kslots = _dims_of(idx, 3, "idx")[2]
    _expect(idx, (B, Lq, kslots), "idx")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, Lq, Hq, device=q.device, dtype=torch.float32)
    _expect(out, (B, Lq, Hq, d), "out")
    _expect(lse, (B, Lq, Hq), "lse")
    if ws is None:
        nbytes = sparse_attn_unique_workspace_bytes(B, Lq, Lk, q_offset, Hq, d, kslots)
        ws = torch.empty(max(nbytes, 1), device=q.device, dtype=torch.uint8) if nbytes else None
    nws = 0 if ws is None else ws.numel() * ws.element_size()
    rc = _lib.ic_sparse_attn_unique(_ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                                    _ptr(v, torch.bfloat16, "v"), _ptr(idx, torch.int32, "idx"),
                                    B, Lq, Lk, Hq, Hkv, d, kslots, q_offset, float(scale),
                                    _ptr(out, torch.bfloat16, "out"),
                                    _ptr(lse, torch.float32, "lse"),
                                    _ptr(ws, None, "ws") if nws else None, nws, _stream(stream))
    _check(rc, "ic_sparse_attn_unique")
    return out, lse


def sparse_attn_no_alloc(q, k, v, idx, q_offset: int = 0, scale: float = 0.0, out=None,
                         lse=None, want_lse: bool = True, stream=None):
    """ic_sparse_attn_no_alloc: the same attention without a workspace.

    For callers that cannot hand the library device memory of its own (see
    include/indexcache.h): split partials live in the library's fixed 4 MiB
    device array; calls that overlap on the GPU race on it.
    """
    B, Lq, Hq, d, Lk, Hkv = _kv_shapes(q, k, v)
    kslots = _dims_of(idx, 3, "idx")[2]
    _expect(idx, (B, Lq, kslots), "idx")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, Lq, Hq, device=q.device, dtype=torch.float32)
    _expect(out, (B, Lq, Hq, d), "out")
    _expect(lse, (B, Lq, Hq), "lse")
    rc = _lib.ic_sparse_attn_no_alloc(_ptr(q, torch.bfloat16, "q"), _ptr(k, torch.bfloat16, "k"),
                                      _ptr(v, torch.bfloat16, "v"), _ptr(idx, torch.int32, "idx"),
                                      B, Lq, Lk, Hq, Hkv, d, kslots, q_offset, float(scale),
                                      _ptr(out, torch.bfloat16, "out"),
                                      _ptr(lse, torch.float32, "lse"), _stream(stream))
    _check(rc, "ic_sparse_attn_no_alloc")
    return out, lse


def make_dims(B, Lq, Lk, q_offset, H_I, d_I, Hq, d, k, scale=0.0, Hkv=1) -> ICDims:
    return ICDims(B, Lq, Lk, q_offset, H_I, d_I, Hq, Hkv, d, k, float(scale))


def layer_stack_workspace_bytes(dims: ICDims, n_layers: int, rows_per_chunk: int = 0) -> int:
    return int(_lib.ic_layer_stack_workspace_bytes(ctypes.byref(dims), n_layers, rows_per_chunk))


def layer_stack_dense_rows(dims: ICDims, ws_bytes: int) -> int:
    """Rows per sequence the stack sends to the dense-masked attention."""
    return int(_lib.ic_layer_stack_dense_rows(ctypes.byref(dims), int(ws_bytes)))


class LayerStack:
    """Holds the C layer table for repeated ic_layer_stack_forward calls.

    layers: per layer a dict with 'q','k','v' (and 'q_idx','k_idx','w' for F
    layers) CUDA tensors; outputs are allocated once here.  fused_topk / z
    are the ic_stack_options fields (None: the library's defaults).
    """

    def __init__(self, pattern: str, layers: Sequence[dict], dims: ICDims, *, want_lse=False,
                 dump_idx=False, ws_bytes: Optional[int] = None, rows_per_chunk: int = 0,
                 fused_topk: Optional[int] = None, z: float = 0.0):
        self.pattern = pattern
        self.dims = dims
        self.opts = None if fused_topk is None and not z else ICStackOptions(
            -1 if fused_topk is None else int(fused_topk), float(z))
        n = len(layers)
        d = dims
        for i, L in enumerate(layers):
            _expect(L["q"], (d.B, d.Lq, d.Hq, d.d), f"layer {i} q")
            kv = (d.B, d.Lk, d.Hkv, d.d) if L["k"].dim() == 4 else (d.B, d.Lk, d.d)
            _expect(L["k"], kv, f"layer {i} k")
            _expect(L["v"], kv, f"layer {i} v")
            if i < len(pattern) and pattern[i] in "F1":
                for name, shape in (("q_idx", (d.B, d.Lq, d.H_I, d.d_I)),
                                    ("k_idx", (d.B, d.Lk, d.d_I)), ("w", (d.B, d.Lq, d.H_I))):
                    if L.get(name) is None:
                        raise ValueError(f"layer {i} is a full layer but has no {name}")
                    _expect(L[name], shape, f"layer {i} {name}")
        dev = layers[0]["q"].device
        self.layers = list(layers)
        self.outs = [torch.empty_like(L["q"]) for L in layers]
        self.lses = [torch.empty(dims.B, dims.Lq, dims.Hq, device=dev, dtype=torch.float32)
                     if want_lse else None for _ in layers]
        self.dumps = [torch.empty(dims.B, dims.Lq, dims.k, device=dev, dtype=torch.int32)
                      if dump_idx else None for _ in layers]
        self.idx_cache = torch.empty(dims.B, dims.Lq, dims.k, device=dev, dtype=torch.int32)
        if ws_bytes is None:
            ws_bytes = layer_stack_workspace_bytes(dims, n, rows_per_chunk)
        self.ws = torch.empty(max(int(ws_bytes), 16), device=dev, dtype=torch.uint8)
        self.table = (ICLayer * n)()
        for i, L in enumerate(layers):
            full = pattern[i] in "F1" if i < len(pattern) else False
            self.table[i] = ICLayer(
                _ptr(L["q"], torch.bfloat16, "q"), _ptr(L["k"], torch.bfloat16, "k"),
                _ptr(L["v"], torch.bfloat16, "v"),
                _ptr(L.get("q_idx"), torch.bfloat16, "q_idx") if full else None,
                _ptr(L.get("k_idx"), torch.bfloat16, "k_idx") if full else None,
                _ptr(L.get("w"), torch.float32, "w") if full else None,
                _ptr(self.outs[i], torch.bfloat16, "out"),
                _ptr(self.lses[i], torch.float32, "lse"), _ptr(self.dumps[i], torch.int32, "dump"))
        self._pattern_b = pattern.encode()

    def forward(self, stream=None, events=None):
        """Runs the stack; `events` (a ctypes array of MARKS_PER_LAYER*n_layers
        cudaEvent_t handles, or None) selects ic_layer_stack_forward_events."""
        if self.opts is not None:
            if events is not None and len(events) < MARKS_PER_LAYER * len(self.layers):
                raise ValueError(f"events holds {len(events)} handles, the stack records "
                                 f"{MARKS_PER_LAYER * len(self.layers)}")
            rc = _lib.ic_layer_stack_forward_opts(
                self._pattern_b, len(self.layers), self.table, ctypes.byref(self.dims),
                ctypes.byref(self.opts), _ptr(self.idx_cache), _ptr(self.ws), self.ws.numel(),
                _stream(stream), None if events is None else ctypes.cast(events, ctypes.c_void_p))
        elif events is None:
            rc = _lib.ic_layer_stack_forward(self._pattern_b, len(self.layers), self.table,
                                             ctypes.byref(self.dims), _ptr(self.idx_cache),
                                             _ptr(self.ws), self.ws.numel(), _stream(stream))
        else:
            need = MARKS_PER_LAYER * len(self.layers)
            if len(events) < need:
                raise ValueError(f"events holds {len(events)} handles, the stack records {need}")
            rc = _lib.ic_layer_stack_forward_events(
                self._pattern_b, len(self.layers), self.table, ctypes.byref(self.dims),
                _ptr(self.idx_cache), _ptr(self.ws), self.ws.numel(), _stream(stream),
                ctypes.cast(events, ctypes.c_void_p))
        _check(rc, "ic_layer_stack_forward")
        return self.outs

    def fused_fallback_blocks(self, stream=None) -> int:
        """Query blocks of the last F layer's last chunk that the fused top-k
        re-ran on the plain path (synchronises the stream)."""
        out = ctypes.c_int(0)
        rc = _lib.ic_layer_stack_fused_fallback_blocks(
            ctypes.byref(self.dims), None if self.opts is None else ctypes.byref(self.opts),
            _ptr(self.ws), self.ws.numel(), _stream(stream), ctypes.byref(out))
        _check(rc, "ic_layer_stack_fused_fallback_blocks")
        return int(out.value)


def layer_stack_forward(pattern: str, layers: Sequence[dict], dims: ICDims, **kw):
    """One-shot helper: builds a LayerStack and runs it once."""
    st = LayerStack(pattern, layers, dims, **kw)
    st.forward()
    return st
