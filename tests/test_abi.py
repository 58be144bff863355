"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/indexcache.h declares, and rejects bad arguments
before launching anything."""
import ctypes
import os
import re

import pytest
from hypothesis import given, settings, strategies as st

from lightning_indexer_top_relu_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "indexcache.h")


@pytest.fixture(scope="module")
def ic():
    build.build()
    from lightning_indexer_top_relu_b200 import indexcache
    return indexcache


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(ic_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_four_steps():
    names = declared_functions()
    for n in ("ic_indexer_scores", "ic_topk_select", "ic_sparse_attn", "ic_layer_stack_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(ic):
    lib = ctypes.CDLL(ic.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(ic.EXPORTS) <= set(declared_functions())


def test_status_strings(ic):
    lib = ic.lib()
    for code, name in ic.STATUS.items():
        assert lib.ic_status_string(code).decode() == name


def _dims(ic, **kw):
    base = dict(B=1, Lq=64, Lk=64, q_offset=0, H_I=4, d_I=64, Hq=8, d=64, k=8)
    base.update(kw)
    return ic.make_dims(**base)


def _stack_call(ic, pattern, dims, n_layers=None, table=None):
    n = len(pattern) if n_layers is None else n_layers
    if table is None:
        table = (ic.ICLayer * max(n, 1))()
        for i in range(max(n, 1)):
            # fake, 16-byte aligned non-null device addresses: validation must
            # reject the call before anything dereferences them
            table[i] = ic.ICLayer(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 0x7000, None, None)
    return ic.lib().ic_layer_stack_forward(pattern.encode(), n, table, ctypes.byref(dims), 0x8000,
                                           0x9000, 1 << 20, None)


def test_leading_shared_layer_is_rejected_before_launch(ic):
    d = _dims(ic)
    assert _stack_call(ic, "SFSS", d) == 3          # IC_ERR_NO_CACHED_INDICES
    assert _stack_call(ic, "0111", d) == 3
    assert b"Shared" in ic.lib().ic_last_error_message()


def test_bad_pattern_and_lengths(ic):
    d = _dims(ic)
    assert _stack_call(ic, "FXSS", d) == 1
    assert _stack_call(ic, "FSS", d, n_layers=4) == 1   # strlen != n_layers
    assert _stack_call(ic, "F", d, n_layers=0) == 1


def test_unsupported_shapes(ic):
    assert _stack_call(ic, "FS", _dims(ic, d_I=96)) == 2
    assert _stack_call(ic, "FS", _dims(ic, H_I=6)) == 2
    assert _stack_call(ic, "FS", _dims(ic, d=80)) == 2
    assert _stack_call(ic, "FS", _dims(ic, Hq=12)) == 2
    d = _dims(ic)
    d.Hkv = 2
    assert _stack_call(ic, "FS", d) == 2


def test_bad_sizes(ic):
    assert _stack_call(ic, "FS", _dims(ic, k=0)) == 1
    assert _stack_call(ic, "FS", _dims(ic, k=65)) == 1          # k > Lk
    assert _stack_call(ic, "FS", _dims(ic, Lq=64, Lk=32)) == 1   # q_offset + Lq > Lk
    assert _stack_call(ic, "FS", _dims(ic, q_offset=-1)) == 1
    lib = ic.lib()
    assert lib.ic_topk_select(0x1000, 1, 4, 4, 0, 0, 0x2000, None) == 1       # k = 0
    assert lib.ic_indexer_scores(None, 0x1000, 0x2000, 1, 4, 4, 4, 64, 0, 0x3000, None) == 1
    assert lib.ic_indexer_scores(0x1008, 0x1000, 0x2000, 1, 4, 4, 4, 64, 0, 0x3000, None) == 2
    assert lib.ic_sparse_attn(0x1000, 0x1000, 0x1000, 0x1000, 1, 4, 4, 8, 1, 64, 0, 0, 0.0,
                              0x1000, None, None, 0, None) == 1             # k = 0


def test_null_layer_tensors(ic):
    table = (ic.ICLayer * 2)()
    table[0] = ic.ICLayer(0x1000, 0x2000, 0x3000, None, 0x5000, 0x6000, 0x7000, None, None)
    table[1] = ic.ICLayer(0x1000, 0x2000, 0x3000, None, None, None, 0x7000, None, None)
    assert _stack_call(ic, "FS", _dims(ic), table=table) == 1   # F layer without q_idx
    table[0] = ic.ICLayer(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 0x7000, None, None)
    table[1] = ic.ICLayer(0x1000, None, 0x3000, None, None, None, 0x7000, None, None)
    assert _stack_call(ic, "FS", _dims(ic), table=table) == 1   # missing k


def test_workspace_query(ic):
    d = _dims(ic, Lq=512, Lk=512, H_I=4)
    full = ic.layer_stack_workspace_bytes(d, 4)
    assert full >= 512 * 512 * 4
    one_block = ic.layer_stack_workspace_bytes(d, 4, rows_per_chunk=1)
    assert 0 < one_block < full
    assert ic.layer_stack_workspace_bytes(_dims(ic, d_I=96), 4) == 0


def test_rejected_calls_launch_nothing(ic):
    before = ic.kernel_launch_count()
    assert _stack_call(ic, "SF", _dims(ic)) == 3                   # leading S
    assert _stack_call(ic, "FX", _dims(ic)) == 1                   # bad pattern character
    assert ic.kernel_launch_count() == before


def test_marks_per_layer_matches_header(ic):
    text = open(HEADER).read()
    m = re.search(r"#define\s+IC_MARKS_PER_LAYER\s+(\d+)", text)
    assert m and int(m.group(1)) == ic.MARKS_PER_LAYER


def test_index_overlap_rejects_bad_sizes_before_launch(ic):
    lib = ic.lib()
    before = ic.kernel_launch_count()
    assert lib.ic_index_overlap(0x1000, 0x1000, 4, 0, 100, 0x2000, None) == 1     # k = 0
    assert lib.ic_index_overlap(0x1000, 0x1000, -1, 8, 100, 0x2000, None) == 1    # n_rows < 0
    assert lib.ic_index_overlap(0x1000, 0x1000, 4, 8, 0, 0x2000, None) == 2       # Lk = 0
    assert lib.ic_index_overlap(0x1000, 0x1000, 4, 8, 1 << 19, 0x2000, None) == 2 # Lk too large
    assert lib.ic_index_overlap(None, 0x1000, 4, 8, 100, 0x2000, None) == 1       # null
    assert lib.ic_index_overlap(None, None, 0, 8, 100, None, None) == 0           # nothing to do
    assert ic.kernel_launch_count() == before


def test_layer_stack_dense_rows(ic):
    """Rows t < 6k, whole blocks of 128/Hq queries, d = 128, with a workspace
    that holds the bitmask, one block of scores and V^T; 0 otherwise."""
    def rows(ws=None, **kw):
        d = dict(B=1, Lq=700, Lk=700, q_offset=0, H_I=32, d_I=128, Hq=16, d=128, k=96)
        d.update(kw)
        dims = ic.make_dims(d["B"], d["Lq"], d["Lk"], d["q_offset"], d["H_I"], d["d_I"], d["Hq"],
                            d["d"], d["k"])
        if ws is None:
            ws = ic.layer_stack_workspace_bytes(dims, 2)
        return ic.layer_stack_dense_rows(dims, ws)
    assert rows() == 576                       # min(6k, L) = 576 -> 72 blocks of 8
    assert rows(k=48) == 288                   # 6k = 288
    assert rows(k=128) == 696                  # min(6k, L) = 700 -> 87 blocks of 8
    assert rows(k=128, Hq=8) == 688            # blocks of 16 queries
    assert rows(d=64, Hq=8) == 0               # the dense kernel needs d = 128
    assert rows(Lq=1, Lk=32768, q_offset=32767, k=2048) == 0     # decode: t far beyond 6k
    assert rows(Lq=300, Lk=1324, q_offset=1024, k=512) == 296    # mid-sequence chunk
    assert rows(ws=1000) == 0                  # workspace too small: every row gathers
    assert rows(d_I=96) == 0                   # invalid dims


@settings(max_examples=300, deadline=None)
@given(Lq=st.integers(1, 20000), q0=st.integers(0, 70000), extra=st.integers(0, 1000),
       k=st.integers(1, 4096), Hq=st.sampled_from([1, 2, 4, 8, 16, 32, 64, 128, 12, 48]),
       d=st.sampled_from([64, 128]), B=st.integers(1, 3), rpc=st.sampled_from([0, 1, 200]))
def test_layer_stack_dense_rows_rule_and_own_workspace(ic, Lq, q0, extra, k, Hq, d, B, rpc):
    """The rule as stated (rows t < 6k, at most 65536 visible keys, whole
    blocks of 128/Hq queries, d = 128) holds on random shapes, and the size
    the workspace query returns always lets the stack take the dense path,
    whatever the score chunking."""
    Lk = q0 + Lq + extra
    k = min(k, Lk)
    dims = ic.make_dims(B, Lq, Lk, q0, 32, 128, Hq, d, k)
    if d != 128 or 128 % Hq:
        want = 0
    else:
        qbd = 128 // Hq
        lim = min(6 * k - q0, 65536 - q0, Lq)
        want = lim // qbd * qbd if lim >= qbd else 0
    ws = ic.layer_stack_workspace_bytes(dims, 2, rpc)
    assert ws > 0
    assert ic.layer_stack_dense_rows(dims, ws) == want
    assert ic.layer_stack_dense_rows(dims, 0) == 0
    # a smaller score chunk never asks for more workspace
    if rpc:
        assert ws <= ic.layer_stack_workspace_bytes(dims, 2, 0)


def test_unique_attention_rejects_bad_arguments_before_launch(ic):
    lib = ic.lib()
    f = lib.ic_sparse_attn_unique
    before = ic.kernel_launch_count()
    ok = dict(q=0x1000, k=0x2000, v=0x3000, idx=0x4000, B=1, Lq=64, Lk=64, Hq=16, Hkv=1, d=128,
              ks=32, q0=0, scale=0.0, out=0x5000, lse=None, ws=None, wsb=0)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["q"], a["k"], a["v"], a["idx"], a["B"], a["Lq"], a["Lk"], a["Hq"], a["Hkv"],
                 a["d"], a["ks"], a["q0"], a["scale"], a["out"], a["lse"], a["ws"], a["wsb"], None)
    assert call(Hkv=2) == 2                      # MQA only
    assert call(ks=0) == 1                       # k < 1
    assert call(q0=10) == 1                      # q_offset + Lq > Lk
    assert call(q=None) == 1                     # null operand
    assert call(k=0x2008) == 2                   # K not 16-byte aligned
    assert call(scale=float("nan")) == 1         # scale not finite
    assert call(wsb=64) == 1                     # workspace size without a workspace
    assert call(B=0) == 0                        # nothing to do
    assert ic.kernel_launch_count() == before


def test_empty_batches_and_rows_are_no_ops(ic):
    """An empty batch or zero query rows is a valid call: every entry point
    returns IC_OK and launches nothing (no device is touched, so this runs
    without a GPU)."""
    lib = ic.lib()
    before = ic.kernel_launch_count()
    for B, Lq, q0 in ((0, 4, 0), (1, 0, 4)):
        assert lib.ic_indexer_scores(0x1000, 0x1000, 0x2000, B, Lq, 4, 4, 64, q0, 0x3000, None) == 0
        assert lib.ic_topk_select(0x1000, B, Lq, 4, q0, 2, 0x2000, None) == 0
        args = (0x1000, 0x1000, 0x1000, 0x1000, B, Lq, 4, 8, 1, 64, 2, q0, 0.0, 0x1000, None)
        assert lib.ic_sparse_attn(*args, None, 0, None) == 0
        assert lib.ic_sparse_attn_no_alloc(*args, None) == 0
        assert lib.ic_sparse_attn_unique(*args, None, 0, None) == 0
        d = _dims(ic, B=B, Lq=Lq, Lk=4, q_offset=q0, k=2)
        assert _stack_call(ic, "FS", d) == 0
    assert lib.ic_index_overlap(0x1000, 0x1000, 0, 8, 16, 0x2000, None) == 0
    assert ic.kernel_launch_count() == before


def test_unique_attention_workspace_query(ic):
    q = ic.sparse_attn_unique_workspace_bytes
    assert q(1, 700, 700, 0, 16, 128, 96) > 700 * 12 * 4        # bitmask + V^T at least
    assert q(0, 700, 700, 0, 16, 128, 96) == 0
    assert q(1, 700, 600, 0, 16, 128, 96) == 0                  # q_offset + Lq > Lk


def test_misaligned_buffers_are_rejected_before_launch(ic):
    """Every buffer a kernel reads with vector, bulk or TMA copies must be
    16-byte aligned (bf16 tensors, w, the workspaces), every fp32 / int32
    buffer 4-byte aligned: otherwise IC_ERR_UNSUPPORTED (2), not a device fault."""
    lib = ic.lib()
    before = ic.kernel_launch_count()
    U = 2

    def indexer(**kw):
        a = dict(q=0x1000, k=0x2000, w=0x3000, s=0x4000)
        a.update(kw)
        return lib.ic_indexer_scores(a["q"], a["k"], a["w"], 1, 64, 64, 4, 64, 0, a["s"], None)
    assert indexer(w=0x3004) == U                # head weights feed a 16-byte bulk copy
    assert indexer(s=0x4002) == U
    assert indexer(q=0x1008) == U

    def topk(**kw):
        a = dict(s=0x1000, i=0x2000)
        a.update(kw)
        return lib.ic_topk_select(a["s"], 1, 64, 64, 0, 8, a["i"], None)
    assert topk(s=0x1002) == U and topk(i=0x2001) == U

    attn_ok = dict(q=0x1000, k=0x2000, v=0x3000, idx=0x4000, out=0x5000, lse=None, ws=None, wsb=0)

    def attn(f, with_ws, **kw):
        a = dict(attn_ok)
        a.update(kw)
        head = (a["q"], a["k"], a["v"], a["idx"], 1, 64, 64, 16, 1, 128, 32, 0, 0.0, a["out"],
                a["lse"])
        return f(*head, a["ws"], a["wsb"], None) if with_ws else f(*head, None)
    for f, with_ws in ((lib.ic_sparse_attn, True), (lib.ic_sparse_attn_unique, True),
                       (lib.ic_sparse_attn_no_alloc, False)):
        assert attn(f, with_ws, out=0x5008) == U     # the dense-masked kernel stores 16 bytes
        assert attn(f, with_ws, idx=0x4002) == U
        assert attn(f, with_ws, lse=0x6002) == U
        if with_ws:
            assert attn(f, with_ws, ws=0x7008, wsb=1 << 16) == U

    assert lib.ic_index_overlap(0x1000, 0x2000, 4, 8, 100, 0x3002, None) == U
    assert lib.ic_index_overlap(0x1001, 0x2000, 4, 8, 100, 0x3000, None) == U

    d = _dims(ic)
    layer = dict(q=0x1000, k=0x2000, v=0x3000, q_idx=0x4000, k_idx=0x5000, w=0x6000, out=0x7000,
                 lse=None)

    def stack(idx_cache=0x8000, ws=0x9000, **kw):
        a = dict(layer)
        a.update(kw)
        table = (ic.ICLayer * 2)()
        for i in range(2):
            table[i] = ic.ICLayer(a["q"], a["k"], a["v"], a["q_idx"], a["k_idx"], a["w"], a["out"],
                                  a["lse"], None)
        return lib.ic_layer_stack_forward(b"FS", 2, table, ctypes.byref(d), idx_cache, ws, 1 << 20,
                                          None)
    assert stack(w=0x6004) == U
    assert stack(out=0x7008) == U
    assert stack(lse=0x8002) == U
    assert stack(idx_cache=0x8002) == U
    assert stack(ws=0x9008) == U
    assert ic.kernel_launch_count() == before


def test_binding_rejects_inconsistent_shapes_before_the_library(ic):
    """The C layer sees pointers and sizes only, so the binding checks every
    tensor against the sizes it derives from the leading operand; these CPU
    tensors never reach the library (a consistent call fails later, on the
    device check)."""
    import torch
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    q_idx, k_idx, w = (torch.zeros(1, 8, 4, 64, dtype=bf), torch.zeros(1, 8, 64, dtype=bf),
                       torch.zeros(1, 8, 4, dtype=f32))
    with pytest.raises(ValueError, match="CUDA"):
        ic.indexer_scores(q_idx, k_idx, w)
    with pytest.raises(ValueError, match="k_idx has shape"):
        ic.indexer_scores(q_idx, torch.zeros(1, 8, 32, dtype=bf), w)
    with pytest.raises(ValueError, match="k_idx has shape"):
        ic.indexer_scores(q_idx, torch.zeros(2, 8, 64, dtype=bf), w)
    with pytest.raises(ValueError, match="w has shape"):
        ic.indexer_scores(q_idx, k_idx, torch.zeros(1, 8, 2, dtype=f32))
    with pytest.raises(ValueError, match="out has shape"):
        ic.indexer_scores(q_idx, k_idx, w, out=torch.zeros(1, 8, 7, dtype=f32))
    with pytest.raises(ValueError, match="3 dimensions"):
        ic.topk_select(torch.zeros(8, 8, dtype=f32), 4)
    with pytest.raises(ValueError, match="out has shape"):
        ic.topk_select(torch.zeros(1, 8, 8, dtype=f32), 4, out=torch.zeros(1, 8, 3, dtype=i32))

    q, kv = torch.zeros(1, 8, 16, 128, dtype=bf), torch.zeros(1, 8, 1, 128, dtype=bf)
    idx = torch.zeros(1, 8, 4, dtype=i32)
    for f in (ic.sparse_attn, ic.sparse_attn_unique, ic.sparse_attn_no_alloc):
        with pytest.raises(ValueError, match="CUDA"):
            f(q, kv, kv, idx)
        with pytest.raises(ValueError, match="v has shape"):
            f(q, kv, torch.zeros(1, 9, 1, 128, dtype=bf), idx)
        with pytest.raises(ValueError, match="k has shape"):
            f(q, torch.zeros(1, 8, 1, 64, dtype=bf), kv, idx)
        with pytest.raises(ValueError, match="idx has shape"):
            f(q, kv, kv, torch.zeros(1, 7, 4, dtype=i32))
        with pytest.raises(ValueError, match="out has shape"):
            f(q, kv, kv, idx, out=torch.zeros(1, 8, 8, 128, dtype=bf))
        with pytest.raises(ValueError, match="lse has shape"):
            f(q, kv, kv, idx, lse=torch.zeros(1, 8, 8, dtype=f32))
    with pytest.raises(ValueError, match="counts has shape"):
        ic.index_overlap(idx, idx, 8, counts=torch.zeros(7, 3, dtype=i32))

    dims = ic.make_dims(1, 8, 8, 0, 4, 64, 16, 128, 4)
    full = {"q": q, "k": kv, "v": kv, "q_idx": q_idx, "k_idx": k_idx, "w": w}
    with pytest.raises(ValueError, match="layer 1 w has shape"):
        ic.LayerStack("FF", [full, dict(full, w=torch.zeros(1, 8, 8, dtype=f32))], dims)
    with pytest.raises(ValueError, match="has no k_idx"):
        ic.LayerStack("FF", [full, {n: t for n, t in full.items() if n != "k_idx"}], dims)
    with pytest.raises(ValueError, match="layer 0 q has shape"):
        ic.LayerStack("F", [dict(full, q=torch.zeros(1, 8, 8, 128, dtype=bf))], dims)
    with pytest.raises(ValueError, match="CUDA"):             # S layers need no indexer inputs
        ic.LayerStack("FS", [full, {"q": q, "k": kv, "v": kv}], dims)


def _opts_call(ic, dims, fused, z=0.0, pattern="FS"):
    n = len(pattern)
    table = (ic.ICLayer * n)()
    for i in range(n):
        table[i] = ic.ICLayer(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, 0x7000, None, None)
    opts = ic.ICStackOptions(fused, z)
    return ic.lib().ic_layer_stack_forward_opts(pattern.encode(), n, table, ctypes.byref(dims),
                                                ctypes.byref(opts), 0x8000, 0x9000, 1 << 20,
                                                None, None)


def test_stack_options_are_checked_before_launch(ic):
    before = ic.kernel_launch_count()
    d = _dims(ic)
    assert _opts_call(ic, d, 2) == 1                      # fused_topk outside {-1, 0, 1}
    assert _opts_call(ic, d, -2) == 1
    assert _opts_call(ic, d, 1, z=float("nan")) == 1
    assert _opts_call(ic, d, 1, pattern="SF") == 3        # leading S still found first
    big_k = _dims(ic, Lq=8192, Lk=8192, k=4097)
    assert _opts_call(ic, big_k, 1) == 2                  # the fused top-k needs k <= 4096
    long = _dims(ic, Lq=64, Lk=262145, q_offset=262081)
    assert _opts_call(ic, long, 1) == 2                   # ... and Lk <= 262144
    assert ic.kernel_launch_count() == before


def test_fused_fallback_query_rejects_unfused_dims(ic):
    d = _dims(ic)
    out = ctypes.c_int(-1)
    off = ic.ICStackOptions(0, 0.0)
    rc = ic.lib().ic_layer_stack_fused_fallback_blocks(ctypes.byref(d), ctypes.byref(off), 0x9000,
                                                       1 << 20, None, ctypes.byref(out))
    assert rc == 1 and out.value == -1
    assert ic.lib().ic_layer_stack_fused_fallback_blocks(ctypes.byref(d), None, None, 0, None,
                                                         ctypes.byref(out)) == 1


def test_workspace_holds_the_fused_chunk(ic):
    """At 64K the workspace of one chunk of all rows holds the fused path's
    candidate lists (3k per row, 8 bytes each) and sampled scores."""
    d = _dims(ic, Lq=65536, Lk=65536, H_I=64, d_I=128, Hq=16, d=128, k=2048)
    full = ic.layer_stack_workspace_bytes(d, 8)
    assert full >= 65536 * 3 * 2048 * 8
    # a chunk of 4 query blocks still holds a fused chunk
    assert ic.layer_stack_workspace_bytes(d, 8, rows_per_chunk=16) >= 16 * 3 * 2048 * 8


def test_binding_fails_loudly_without_the_library(tmp_path):
    """No CPU fallback: a copy of the package whose library was never built
    cannot be imported, and neither can the GPU backends that reach the
    library through it."""
    import shutil
    import subprocess
    import sys
    pkg = build.PKG
    dst = tmp_path / os.path.basename(pkg)
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc"))
    name = os.path.basename(pkg)
    env = dict(os.environ, PYTHONPATH=str(tmp_path))
    for stmt in (f"import {name}.indexcache",
                 f"from {name}.drift import GpuBackend; GpuBackend([], None)",
                 f"from {name}.sharding import ShardedStack; ShardedStack('F', [], None, 1, 0)"):
        r = subprocess.run([sys.executable, "-c", stmt], env=env, cwd=str(tmp_path),
                           capture_output=True, text=True, timeout=300)
        assert r.returncode != 0, stmt
        assert "no CPU fallback" in r.stderr, (stmt, r.stderr[-500:])
