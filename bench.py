"""Benchmark of the IndexCache sparse-attention layer stack on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill_64k] [--pattern P] [--no-cpu-baseline]
                    [--no-e2e] [--no-all-f] [--no-extras] [--sweep 4,16,64,128]

One step = one pass of the whole hot path over one batch of synthetic input:
the layer loop with the F-layer indexer + top-k and every layer's sparse
attention (ic_layer_stack_forward), inputs resident in HBM.  The default
workload is the 64K-token prefill: B=1, L=65536, 8 layers FSSSFSSS, indexer
64 heads x 128, k=2048, attention 16 query heads / 1 KV head x 128; the same
inputs also run all-F (FFFFFFFF) for the F/S speed-up.

Prints ONE JSON line (rank 0).  `value` is prefill tokens/s over the stack
(B*L*N / max-over-ranks step time).  `kernels` breaks the step down per
kernel from CUDA events recorded on the launching stream inside the timed
steps; `roofline` is for the kernel with the largest share of the step.
`e2e` is the same stack through the public call with pinned host buffers
(inputs copied in and outputs copied out inside the timed region).  On one
GPU the line also carries supplementary points: `sweep_16_layers` (B=1,
L in {4K, 16K, 64K, 128K}, 16 layers all-F vs (FSSS)x4, indexer share of the
step) and `decode_32k` (B=32 over a 32768-token cache, 16 layers).
With N > 1 (torchrun) every rank runs an independent replica of the workload
(the query rows of different sequences never interact), so scaling is weak
and no collective is on the data path; the barrier and the max-over-ranks
reduction of the step time are the only collectives.

--impl reference times the CPU oracle (the plain fp64 restatement used by the
tests) on the host cores, on a bounded sample of query rows of the same
workload, and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import csv
import ctypes
import io
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from lightning_indexer_top_relu_b200 import synth  # noqa: E402

METRIC = "prefill tokens/s over F/S layer stack; indexer TFLOP/s & top-k/attn HBM GB/s"
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    """Roofline denominators: the copy bandwidth and bf16 GEMM rates measured
    on this machine's B200s (MEASURED_PEAKS.json), else an earlier measurement
    on the same pool, labelled "fallback"."""
    fallback = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        out = {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
               "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    except (OSError, ValueError, KeyError, TypeError):
        return fallback
    return out if out["hbm_gbs"] > 0 and out["bf16_tflops"] > 0 else fallback


# ---------------------------------------------------------------- algorithmic work

DA_TILE = 64              # keys per tile of the dense-masked kernel
SFU_PER_CLK_SM = 16       # ex2 results per clock per SM (CUDA arithmetic-throughput table)


def work_per_layer(wl, lq_d: int = 0):
    """Algorithmic flops / bytes of each step of one layer (causal).  The
    first lq_d rows of each sequence take the dense-masked attention (as the
    library reports for the stack's workspace), in blocks of 128/Hq queries."""
    B, Lq, Lk, q0, k = wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.k
    t = np.arange(Lq, dtype=np.float64) + q0
    vis = np.minimum(t + 1, Lk)
    sel_row = np.minimum(vis, k)
    sum_vis = B * vis.sum()                       # sum over rows of visible positions
    rows = B * Lq
    w = {"rows": rows}
    w["indexer_flops"] = 2.0 * wl.H_I * wl.d_I * sum_vis
    # q_I + w read once, k_I once per batch element, causal scores written
    w["indexer_bytes"] = (rows * wl.H_I * wl.d_I * 2 + rows * wl.H_I * 4 + B * Lk * wl.d_I * 2
                          + 4 * sum_vis)
    w["topk_bytes"] = 4 * sum_vis + 4.0 * rows * k
    # fused indexer -> top-k: the F layer's inputs read once and its index
    # rows written; no score is stored
    w["fused_bytes"] = (rows * wl.H_I * wl.d_I * 2 + rows * wl.H_I * 4 + B * Lk * wl.d_I * 2
                        + 4.0 * rows * k)
    qbd = 128 // wl.Hq if lq_d else 0
    # dense-masked rows: useful flops are those of the selected positions;
    # the kernel executes whole 64-key tiles of 128 rows up to each block's last t
    sel_d = B * sel_row[:lq_d].sum()
    w["dense_rows"] = B * lq_d
    w["dense_flops"] = 4.0 * wl.Hq * wl.d * sel_d
    if lq_d:
        t_last = q0 + np.arange(0, lq_d, qbd) + qbd - 1
        tiles = B * np.ceil(np.minimum(t_last + 1, Lk) / DA_TILE).sum()
    else:
        tiles = 0.0
    w["dense_tiles"] = tiles
    w["dense_exec_flops"] = tiles * 4.0 * 128 * DA_TILE * wl.d
    w["dense_exec_exps"] = tiles * 128 * DA_TILE
    # gathered rows: K and V rows of every selected slot + q + out + index rows
    sel_g = B * sel_row[lq_d:].sum()
    rows_g = B * (Lq - lq_d)
    w["gather_rows"] = rows_g
    w["gather_flops"] = 4.0 * wl.Hq * wl.d * sel_g
    w["gather_bytes"] = 4.0 * wl.d * sel_g + 2 * 2.0 * rows_g * wl.Hq * wl.d + 4.0 * rows_g * k
    return w


# ---------------------------------------------------------------- ncu traffic

_KERNEL_SRC = {"sparse_attn": ("sparse_attn_kernel", ("sparse_attn.cuh",)),
               "dense_attn": ("dense_attn_kernel", ("dense_attn.cuh",)),
               "indexer_scores": ("indexer_scores_kernel", ("indexer_scores.cuh", "fused_topk.cuh")),
               "topk_select": ("topk_select_kernel", ("topk_select.cuh",)),
               "fused_select": ("fused_select_kernel", ("fused_topk.cuh",))}


def _read_profile(path, srcs):
    """(dram bytes per launch, units per launch or None) of a committed ncu
    summary, or None when the kernel's sources changed since the capture
    (the summary records a hash of them)."""
    import hashlib
    h = hashlib.sha256()
    for f in tuple(srcs) + ("common.cuh",):
        with open(os.path.join(ROOT, "lightning_indexer_top_relu_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    want = traffic = units = None
    with open(path) as fh:
        for line in fh:
            if line.startswith("source_hash:"):
                want = line.split(":", 1)[1].strip()
            elif line.startswith("dram_bytes_per_launch:"):
                try:
                    traffic = int(line.split(":", 1)[1].strip())
                except ValueError:
                    traffic = None
            elif line.startswith("units_per_launch:"):
                units = float(line.split(":", 1)[1].strip())
    if want != h.hexdigest()[:16] or traffic is None:
        return None
    return traffic, units


def profile_traffic(kernel: str, workload: str, units: float = 0.0):
    """DRAM bytes per launch of `kernel` from the committed ncu summaries:
    the summary of this workload when there is one; otherwise a summary of a
    case of the same kernel and the same kind (decode rows or prefill rows)
    that records its units per launch (query rows), within 4x of this
    launch's, scaled by units / its units -- the full-size workloads are too
    large for a full ncu capture.  Traffic per row differs between regimes
    (decode rows read K/V from HBM, prefill rows from L2), and so does the
    share that does not grow with the rows, so nothing further is scaled:
    (None, None).  Returns (bytes or None, where from)."""
    import glob
    name, srcs = _KERNEL_SRC[kernel]
    path = os.path.join(ROOT, "profiles", f"{name}_{workload}.md")
    if os.path.exists(path):
        got = _read_profile(path, srcs)
        return (got[0], os.path.basename(path)) if got else (None, None)
    if units > 0:
        # the matching capture whose size is nearest (in ratio) to this launch's
        decode = workload.startswith("decode")
        best = None
        for path in sorted(glob.glob(os.path.join(ROOT, "profiles", f"{name}_*.md"))):
            other = os.path.basename(path)[len(name) + 1:-3]
            if other.startswith("decode") != decode:
                continue
            got = _read_profile(path, srcs)
            if got and got[1]:
                dist = abs(math.log(units / got[1]))
                if dist <= math.log(4.0) and (best is None or dist < best[0]):
                    best = (dist, path, got)
        if best:
            _, path, got = best
            return int(got[0] * units / got[1]), (f"{os.path.basename(path)} scaled by "
                                                  f"{units:g} / {got[1]:g} rows")
    return None, None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi every 200 ms
    while the timed region runs; the samples are read through a pipe (a
    thread drains it), so nothing is written to disk."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, cmd=None):
        self.cmd = cmd or ["nvidia-smi", "-i", str(device_index), f"--query-gpu={self.QUERY}",
                           "--format=csv,noheader,nounits", "-lms", "200"]
        self.proc = None
        self.thread = None
        self.lines = []

    def _drain(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._drain, daemon=True)
        self.thread.start()

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait()
        self.thread.join(timeout=5)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for row in csv.reader(list(self.lines)):
            if len(row) < 9:
                continue
            try:
                sm.append(float(row[1]))
                mx = float(row[2])
            except ValueError:
                continue
            for n, v in zip(names, row[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle leg

def row_slice(wl, layers, r, key_cache=None):
    """Host copies of what the oracle needs for flattened query row r: that
    row's query-side tensors and its sequence's keys (a one-row problem at
    q_offset = t, the row's absolute position).  `key_cache` (a dict) keeps
    the host copy of each sequence's K, V and k_I, so a sample of many rows
    copies every key tensor to the host once."""
    b, i = divmod(int(r), wl.Lq)
    out = []
    for l, L in enumerate(layers):
        d = {}
        for key in ("q", "q_idx", "w"):
            if key in L:
                d[key] = L[key][b:b + 1, i:i + 1].contiguous().cpu()
        for key in ("k", "v", "k_idx"):
            if key in L:
                if key_cache is None:
                    d[key] = L[key][b:b + 1].contiguous().cpu()
                else:
                    ck = (l, key, b)
                    if ck not in key_cache:
                        key_cache[ck] = L[key][b:b + 1].contiguous().cpu()
                    d[key] = key_cache[ck]
        out.append(d)
    return out, wl.q_offset + i


def _oracle_rows(wl, pattern, sl, workers):
    """Runs the oracle on prepared one-row problems `sl`, one row per host
    thread (one OpenMP thread each), and returns the wall time."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    def one(item):
        lay, t = item
        oracle.set_num_threads(1)
        oracle.layer_stack(pattern, lay, wl.k, q_offset=t)

    oracle.num_threads()              # loads (building if needed) before the pool starts
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=workers) as ex:
        list(ex.map(one, sl))
    return time.perf_counter() - t0


def host_cores() -> int:
    """Host cores this process may run on.  The oracle legs run one row per
    core with one OpenMP thread each, so a launcher's OMP_NUM_THREADS (torchrun
    sets 1) does not shrink the pool."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def oracle_rows_per_s(wl, pattern, layers, budget_s=15.0, seed=5):
    """Times the oracle on uniformly drawn query rows, one row per host core,
    for about budget_s seconds; returns (rows/s, sample description, cores)."""
    rng = np.random.default_rng(seed)
    total = wl.B * wl.Lq
    workers = host_cores()
    elapsed, done, n = 0.0, 0, workers
    cache = {}
    while elapsed < budget_s and done < total:
        rows = rng.choice(total, size=min(n, total), replace=False)
        sl = [row_slice(wl, layers, r, cache) for r in rows]
        dt = _oracle_rows(wl, pattern, sl, workers)
        elapsed += dt
        done += len(rows)
        rate = len(rows) / max(dt, 1e-9)
        n = int(max(workers, min(total, rate * max(budget_s - elapsed, 0.0))))
    return done / elapsed, (f"{done} uniformly drawn query rows of {total}, each through all "
                            f"{len(pattern)} layers, {elapsed:.1f} s"), workers


def input_bytes(wl, indexer_for_all=True):
    """Bytes of per-layer inputs the stack reads (bf16 q/K/V, indexer q_I/k_I, fp32 w)."""
    n_f = wl.n_layers if indexer_for_all else sum(c in "F1" for c in wl.pattern)
    attn = wl.B * (wl.Lq * wl.Hq * wl.d + 2 * wl.Lk * wl.d) * 2
    idx = wl.B * (wl.Lq * wl.H_I * wl.d_I * 2 + wl.Lk * wl.d_I * 2 + wl.Lq * wl.H_I * 4)
    return wl.n_layers * attn + n_f * idx


def run_reference(args, wl, pattern):
    """The CPU oracle as the reference arm (rank 0 only): each step is a
    bounded, uniformly drawn sample of --ref-rows query rows of the workload,
    each row through every layer of the pattern."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    big = input_bytes(wl, True) > 2 * 2 ** 30
    dev = torch.device("cuda") if (big and torch.cuda.is_available()) else "cpu"
    layers = synth.make_layers(wl, indexer_for_all=any(c in "F1" for c in pattern), device=dev)
    total = wl.B * wl.Lq
    rng = np.random.default_rng(11)
    want = args.ref_rows if args.ref_rows > 0 else (64 if wl.Lk <= 16384 else 32)
    n_rows = max(1, min(total, want))
    workers = host_cores()
    times = []
    cache = {}
    for s in range(args.warmup + args.steps):
        rows = rng.choice(total, size=n_rows, replace=False)
        sl = [row_slice(wl, layers, r, cache) for r in rows]
        dt = _oracle_rows(wl, pattern, sl, workers)
        if s >= args.warmup:                       # warm-up steps are not timed
            times.append(dt)
    sec = float(np.sum(times))
    value = n_rows * args.steps / sec
    sample = (f"{n_rows} uniformly drawn query rows of {total} per step, each through all "
              f"{len(pattern)} layers, on {workers} host cores (no GPU work)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sec / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl, pattern, args),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": workers,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def aggregate_over_ranks(ms_per_step: float, tokens_per_step: float, dist_mod=None, device=None):
    """Whole-job throughput: step time = max over ranks, tokens = sum over ranks.

    Returns (max ms per step, total tokens per step, tokens/s).  With no process
    group (N = 1) the local numbers are returned unchanged.
    """
    if dist_mod is None:
        return ms_per_step, tokens_per_step, tokens_per_step / (ms_per_step / 1e3)
    t = torch.tensor([ms_per_step], dtype=torch.float64, device=device)
    n = torch.tensor([tokens_per_step], dtype=torch.float64, device=device)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    dist_mod.all_reduce(n, op=dist_mod.ReduceOp.SUM)
    ms, tok = float(t.item()), float(n.item())
    return ms, tok, tok / (ms / 1e3)


def cross_layer_overlap(ic, wl, layers, dims, rpc, stream, peaks, n):
    """Untimed: every layer run as F with its index cache dumped, then the
    top-k overlap of each adjacent pair on the device (ic_index_overlap).
    Reports the statistic the pages quote for real models (adjacent layers
    share 70-100% of their selections) for these synthetic inputs, over rows
    with t >= k (earlier rows select every visible position), and the
    overlap kernel's own rate."""
    stack = ic.LayerStack("F" * n, layers, dims, dump_idx=True, rows_per_chunk=rpc)
    stack.forward(stream)
    torch.cuda.synchronize()
    t = np.arange(wl.Lq) + wl.q_offset
    keep = np.tile(t >= wl.k, wl.B)
    ov, jac, times = [], [], []
    counts = None
    for l in range(n - 1):
        a, b = stack.dumps[l], stack.dumps[l + 1]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        counts = ic.index_overlap(a, b, wl.Lk, counts=counts, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
        c = counts.cpu().numpy().astype(np.float64)[keep]
        if len(c):
            ov.append(float(np.mean(c[:, 0] / wl.k)))
            jac.append(float(np.mean(c[:, 0] / (c[:, 1] + c[:, 2] - c[:, 0] + 1e-8))))
    if ic.get_last_device_error() != 0:
        raise RuntimeError("device error in the overlap pass")
    del stack
    ms = float(np.median(times)) if times else 0.0
    nbytes = 2 * 4.0 * wl.B * wl.Lq * wl.k + 12.0 * wl.B * wl.Lq
    out = {"pairs": n - 1, "rows": "t >= k", "ms_per_launch": ms,
           "gbs": nbytes / (ms * 1e-3) / 1e9 if ms > 0 else None}
    if out["gbs"]:
        out["frac_of_hbm"] = out["gbs"] / peaks["hbm_gbs"]
    if ov:
        out.update({"mean_overlap": float(np.mean(ov)), "min_pair_overlap": float(np.min(ov)),
                    "mean_jaccard": float(np.mean(jac))})
    return out


def config_of(wl, pattern, args):
    return {"workload": wl.name, "B": wl.B, "L": wl.Lq, "Lk": wl.Lk, "q_offset": wl.q_offset,
            "layers": wl.n_layers, "pattern": pattern, "H_I": wl.H_I, "d_I": wl.d_I,
            "k": wl.k, "Hq": wl.Hq, "Hkv": 1, "d": wl.d,
            "parallelism": "replicas" if args.gpus > 1 else "single",
            "l2": "flushed (256 MiB write) before every timed step"}


# ---------------------------------------------------------------- GPU leg

def run_row_sharded(args, wl, pattern, ic, dev, world, rank, local, pg):
    """--shard rows: the ranks split ONE workload's query rows (zig-zag row
    chunks of the sequence for B = 1, whole sequences for B > 1); each step
    every rank runs its shard of the stack, with no collective on the data
    path.  value = the workload's tokens / max-over-ranks step time (strong
    scaling).  Only the whole-step time is reported in this mode."""
    from lightning_indexer_top_relu_b200 import sharding
    layers = synth.make_layers(wl, indexer_for_all=False, device=dev)
    torch.cuda.synchronize()
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    stack = sharding.ShardedStack(pattern, layers, dims, world, rank)
    rows_here = sum(ch.nb * ch.n for ch in stack.chunks)
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024 // 4, device=dev, dtype=torch.float32)
    for _ in range(args.warmup):
        stack.forward(stream)
    torch.cuda.synchronize()
    if ic.get_last_device_error() != 0:
        raise RuntimeError("device error during warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    clocks.start()
    launches0 = ic.kernel_launch_count()
    for s in range(args.steps):
        flush.fill_(float(s))
        starts[s].record(stream)
        stack.forward(stream)
        ends[s].record(stream)
    torch.cuda.synchronize()
    launches = ic.kernel_launch_count() - launches0
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    if ic.get_last_device_error() != 0:
        raise RuntimeError("device error during the timed steps")
    local_ms = float(np.mean([starts[s].elapsed_time(ends[s]) for s in range(args.steps)]))
    ms_per_step, tokens, value = aggregate_over_ranks(local_ms, float(rows_here), pg, dev)
    cfg = config_of(wl, pattern, args)
    cfg["parallelism"] = f"rows{world}" if wl.B == 1 else f"sequences{world}"
    cfg["shard_rank0"] = [[ch.b0, ch.nb, ch.i0, ch.n] for ch in sharding.shard(wl.B, wl.Lq, world, 0)]
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Gaussian, correlated layers)", "config": cfg,
            "gpu_launches": int(launches), "roofline": None,
            "note": "row-sharded mode: whole-step time only; the per-kernel breakdown and "
                    "roofline come from the default (replica) mode"}
    if clk is not None:
        line["clocks"] = clk
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- timing helpers

def new_marks(stream, n_layers: int, npl: int):
    """npl CUDA events per layer for ic_layer_stack_forward_events, created
    (recorded once) so their handles exist before the library records them."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(npl * n_layers)]
    for e in evs:  # torch creates the CUDA event on first record
        e.record(stream)
    arr = (ctypes.c_void_p * (npl * n_layers))(*[e.cuda_event for e in evs])
    assert all(arr), "CUDA event handles must exist before they are handed to the library"
    return evs, arr


def time_stack(ic, stack, stream, flush, steps: int, warmup: int, with_marks: bool = True):
    """`warmup` untimed steps, then `steps` steps each timed with CUDA events
    on the launching stream, L2 flushed (a 256 MiB write) before each.
    Returns (per-step ms, per-step timing marks or None)."""
    n = len(stack.layers)
    for _ in range(warmup):
        stack.forward(stream)
    torch.cuda.synchronize()
    marks = [new_marks(stream, n, ic.MARKS_PER_LAYER) for _ in range(steps)] if with_marks else None
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize()
    for s in range(steps):
        flush.fill_(float(s))
        starts[s].record(stream)
        stack.forward(stream, events=marks[s][1] if marks else None)
        ends[s].record(stream)
    torch.cuda.synchronize()
    return [starts[s].elapsed_time(ends[s]) for s in range(steps)], marks


def timed_steps_for(step_ms: float, target_ms: float = 2000.0, lo: int = 20, hi: int = 2000) -> int:
    """Steps of the main timed region: enough for about target_ms (so the
    clock sampler, one sample per 200 ms, sees the region), within [lo, hi]."""
    return int(min(hi, max(lo, math.ceil(target_ms / max(step_ms, 1e-3)))))


def auto_steps(ic, stack, stream, flush, budget_ms: float, lo: int = 2, hi: int = 10) -> int:
    """Timed steps for a supplementary point: enough to fill about budget_ms
    (one untimed probe step gives the step time), clamped to [lo, hi]."""
    ms, _ = time_stack(ic, stack, stream, flush, 1, 1, with_marks=False)
    return int(min(hi, max(lo, math.ceil(budget_ms / max(ms[0], 1e-3)))))


def kernel_times(wl, pattern, marks, steps: int, npl: int, w):
    """Per-launch times (ms) of each kernel group from the stack's marks:
    indexer (mark 0 -> 1), top-k (1 -> 2) on F layers; dense-masked attention
    (2 -> 3) and gathered attention (3 -> 4) on every layer that has such rows."""
    ki = {"indexer": [], "topk": [], "attn_dense": [], "attn_gather": []}
    for evs, _ in marks:
        for l, c in enumerate(pattern):
            e = evs[npl * l: npl * (l + 1)]
            if c in "F1":
                ki["indexer"].append(e[0].elapsed_time(e[1]))
                ki["topk"].append(e[1].elapsed_time(e[2]))
            if w["dense_rows"]:
                ki["attn_dense"].append(e[2].elapsed_time(e[3]))
            if w["gather_rows"]:
                ki["attn_gather"].append(e[3].elapsed_time(e[4]))
    return {k: v for k, v in ki.items() if v}


def kernel_breakdown(ki, w, steps: int, ms_per_step: float, peaks, sm_mhz: float, n_sms: int,
                     fused: bool = False):
    """Per-kernel rates and shares of the step from kernel_times() output.
    `fused`: the stack fused the top-k into the indexer (the indexer group
    then covers the sampled pass, the thresholds and the candidate pass, and
    the top-k group the exact selection and the fallback rounds)."""
    kernels, per_step = {}, {}
    for name, vals in ki.items():
        avg = float(np.mean(vals))
        sec = avg * 1e-3
        per_step[name] = float(np.sum(vals)) / steps
        ent = {"launches_per_step": len(vals) // steps, "ms_per_launch": avg,
               "share": per_step[name] / ms_per_step}
        if name == "indexer":
            if fused:
                ent["covers"] = ("fused indexer: sampled key tiles + per-row thresholds + the "
                                 "candidate pass (no score stored); tflops counts the flops of "
                                 "every visible score once")
            ent["tflops"] = w["indexer_flops"] / sec / 1e12
            ent["frac_of_bf16_peak"] = ent["tflops"] / peaks["bf16_tflops"]
            if peaks.get("bf16_tflops_sustained"):
                ent["frac_of_bf16_sustained"] = ent["tflops"] / peaks["bf16_tflops_sustained"]
            ent["gbs"] = w["indexer_bytes"] / sec / 1e9
        elif name == "topk" and fused:
            ent["covers"] = ("exact selection over the candidate lists (also writes the selection "
                             "bitmask of dense-masked rows) + the fallback rounds")
        elif name == "topk":
            ent["covers"] = "top-k select (also writes the selection bitmask of dense-masked rows)"
            ent["gbs"] = w["topk_bytes"] / sec / 1e9
            ent["frac_of_hbm"] = ent["gbs"] / peaks["hbm_gbs"]
        elif name == "attn_dense":
            ent["covers"] = "V transpose + dense-masked tcgen05 attention, rows t < 6k"
            ent["rows"] = int(w["dense_rows"])
            ent["tflops"] = w["dense_flops"] / sec / 1e12
            ent["frac_of_bf16_peak"] = ent["tflops"] / peaks["bf16_tflops"]
            ent["executed_tflops"] = w["dense_exec_flops"] / sec / 1e12
            ent["executed_frac_of_bf16_peak"] = ent["executed_tflops"] / peaks["bf16_tflops"]
            sfu_peak = SFU_PER_CLK_SM * n_sms * sm_mhz * 1e6
            ent["exp2_per_s"] = w["dense_exec_exps"] / sec
            ent["frac_of_sfu_peak"] = ent["exp2_per_s"] / sfu_peak
        else:
            ent["covers"] = "gather attention (+ split combine), rows t >= 6k"
            ent["rows"] = int(w["gather_rows"])
            ent["tflops"] = w["gather_flops"] / sec / 1e12
            ent["logical_gbs"] = w["gather_bytes"] / sec / 1e9
            ent["frac_of_hbm"] = ent["logical_gbs"] / peaks["hbm_gbs"]
        kernels[name] = ent
    return kernels, per_step


def tensor_peak(peaks, clk):
    """The bf16 denominator for a contraction timed inside the step: the
    sustained (power-capped) cuBLAS rate when the clock record shows the SM
    clock held down by the power cap (sw_power_cap active, or the median SM
    clock under load below 95% of its maximum), else the burst rate.
    Returns (peak, which)."""
    sus = peaks.get("bf16_tflops_sustained")
    capped = False
    if clk:
        mx = clk.get("sm_max_mhz") or 0.0
        capped = "sw_power_cap" in clk.get("reasons", []) or (
            mx > 0 and clk.get("sm_mhz", mx) < 0.95 * mx)
    if capped and sus:
        return float(sus), "sustained"
    return float(peaks["bf16_tflops"]), "burst"


def roofline_of(kernels, w, peaks, clk, workload: str):
    """Roofline entry for the kernel with the largest share of the step."""
    dom = max(kernels, key=lambda k: kernels[k]["share"])
    kd = kernels[dom]
    tpeak, tkind = tensor_peak(peaks, clk)
    if dom == "indexer":
        roof = {"kernel": "indexer_scores", "bound": "tensor", "achieved": kd["tflops"],
                "peak": tpeak, "peak_kind": tkind, "unit": "TFLOP/s",
                "frac": kd["tflops"] / tpeak,
                "frac_of_burst": kd["tflops"] / peaks["bf16_tflops"],
                "algorithmic_per_launch": w["indexer_flops"],
                "note": "achieved = 2*H_I*d_I flops per (query, visible key) / event time"}
    elif dom == "topk" and "gbs" not in kd:
        roof = {"kernel": "fused_select", "bound": "latency", "achieved": None, "peak": None,
                "unit": None, "frac": None}
    elif dom == "topk":
        roof = {"kernel": "topk_select", "bound": "hbm", "achieved": kd["gbs"],
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": kd["gbs"] / peaks["hbm_gbs"],
                "algorithmic_per_launch": w["topk_bytes"]}
    elif dom == "attn_dense":
        roof = {"kernel": "dense_attn", "bound": "tensor", "achieved": kd["tflops"],
                "peak": tpeak, "peak_kind": tkind, "unit": "TFLOP/s",
                "frac": kd["tflops"] / tpeak,
                "frac_of_burst": kd["tflops"] / peaks["bf16_tflops"],
                "algorithmic_per_launch": w["dense_flops"],
                "executed_frac": kd["executed_tflops"] / tpeak,
                "sfu_frac": kd["frac_of_sfu_peak"],
                "note": ("achieved counts the flops of the selected positions only (4*Hq*d per "
                         "slot); the kernel runs whole 64-key tiles, whose flops give "
                         "executed_frac, and one exp2 per tile element on the SFUs "
                         "(16/clk/SM), whose rate gives sfu_frac")}
    else:
        roof = {"kernel": "sparse_attn", "bound": "hbm", "achieved": kd["logical_gbs"],
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": kd["logical_gbs"] / peaks["hbm_gbs"],
                "algorithmic_per_launch": w["gather_bytes"],
                "note": ("achieved counts the logical K/V gather bytes; when a layer's K/V stay "
                         "L2-resident, DRAM traffic (`traffic`) is far below them")}
    roof["peak_source"] = peaks["source"]
    units = {"indexer_scores": w.get("rows", 0), "sparse_attn": w.get("gather_rows", 0),
             "dense_attn": w.get("dense_rows", 0), "topk_select": w.get("rows", 0),
             "fused_select": w.get("rows", 0)}.get(roof["kernel"], 0)
    roof["traffic"], src = (profile_traffic(roof["kernel"], workload, units)
                            if roof["kernel"] in _KERNEL_SRC else (None, None))
    if src:
        roof["traffic_from"] = src
    return roof


def default_rows_per_chunk(wl) -> int:
    """F-layer score rows per chunk: as many as 16 GiB of fp32 scores allow."""
    return max(1, min(wl.B * wl.Lq, (16 * 2 ** 30) // (4 * wl.Lk)))


def fused_state(ic, stack):
    """(fused, fallback blocks): whether the stack fused the top-k into the
    indexer, and how many query blocks of its last F layer's last chunk fell
    back to the plain path (synchronises)."""
    try:
        return True, stack.fused_fallback_blocks()
    except ic.IndexCacheError:
        return False, None


def stack_point(ic, wl, pattern, layers, stream, flush, peaks, n_sms, clk, budget_ms,
                rows_per_chunk=0, warmup=1):
    """One supplementary stack measurement: step time, tokens/s, the indexer
    share of the step and the indexer's tensor rate, from the stack's marks."""
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    rpc = rows_per_chunk or default_rows_per_chunk(wl)
    stack = ic.LayerStack(pattern, layers, dims, rows_per_chunk=rpc)
    lq_d = ic.layer_stack_dense_rows(dims, stack.ws.numel())
    steps = auto_steps(ic, stack, stream, flush, budget_ms)
    ms, marks = time_stack(ic, stack, stream, flush, steps, warmup)
    if ic.get_last_device_error() != 0:
        raise RuntimeError(f"device error in the {wl.name} {pattern} point")
    w = work_per_layer(wl, lq_d)
    msps = float(np.mean(ms))
    fused, fallback = fused_state(ic, stack)
    ki = kernel_times(wl, pattern, marks, steps, ic.MARKS_PER_LAYER, w)
    kern, per_step = kernel_breakdown(ki, w, steps, msps, peaks,
                                      (clk or {}).get("sm_mhz") or 1965.0, n_sms, fused)
    out = {"pattern": pattern, "steps": steps, "ms_per_step": msps, "fused_topk": fused,
           "tokens_per_s": wl.B * wl.Lq / (msps * 1e-3),
           "indexer_share": (per_step.get("indexer", 0) + per_step.get("topk", 0)) / msps}
    if "indexer" in kern:
        out["indexer_ms_per_launch"] = kern["indexer"]["ms_per_launch"]
        out["indexer_tflops"] = kern["indexer"]["tflops"]
        out["indexer_frac_of_bf16_peak"] = kern["indexer"]["frac_of_bf16_peak"]
    if "topk" in kern:
        out["topk_ms_per_launch"] = kern["topk"]["ms_per_launch"]
        if "indexer" in kern and kern["topk"]["ms_per_launch"] < 0.01 * kern["indexer"]["ms_per_launch"]:
            # an F layer run in several workspace chunks interleaves the
            # indexer and the top-k of each chunk: the layer's one indexer
            # span then covers both (its rate is a lower bound)
            out["indexer_span_includes_topk"] = True
    for name in ("attn_dense", "attn_gather"):
        if name in kern:
            out[f"{name}_ms_per_launch"] = kern[name]["ms_per_launch"]
    del stack
    return out


def sweep_points(ic, lengths_k, dev, stream, flush, peaks, n_sms, clk):
    """The indexer + top-k sweep: B = 1, L in lengths (K tokens), indexer
    64 x 128, k = 2048, a 16-layer stack run all-F and (FSSS)x4, each with the
    indexer share of the step.  Inputs are drawn on the device."""
    import dataclasses
    out = {}
    for lk in lengths_k:
        base = synth.WORKLOADS[f"sweep_{lk}k"]
        wl = dataclasses.replace(base, n_layers=16, pattern="FSSS" * 4)
        layers = synth.make_layers(wl, indexer_for_all=True, device=dev)
        torch.cuda.synchronize()
        pt = {}
        for pat in ("F" * 16, "FSSS" * 4):
            pt["all_f" if pat == "F" * 16 else "fsss_x4"] = stack_point(
                ic, wl, pat, layers, stream, flush, peaks, n_sms, clk, budget_ms=1500.0)
        pt["speedup_of_pattern"] = pt["all_f"]["ms_per_step"] / pt["fsss_x4"]["ms_per_step"]
        out[f"{lk}k"] = pt
        del layers
        torch.cuda.empty_cache()
    return out


def graph_point(ic, wl, pattern, layers, flush, steps: int = 20, warmup: int = 3):
    """The same stack replayed from a CUDA graph (one forward captured after
    warm-up): the launches of a step are submitted at once, so small steps
    (decode) lose the gaps between kernel launches.  The library issues no
    host synchronisation inside a forward, which is what makes it capturable."""
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    stack = ic.LayerStack(pattern, layers, dims, rows_per_chunk=default_rows_per_chunk(wl))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(warmup):
            stack.forward(side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        stack.forward()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    for s in range(steps):
        flush.fill_(float(s))
        starts[s].record(st)
        g.replay()
        ends[s].record(st)
    torch.cuda.synchronize()
    if ic.get_last_device_error() != 0:
        raise RuntimeError(f"device error in the {wl.name} graph replay")
    ms = float(np.mean([a.elapsed_time(b) for a, b in zip(starts, ends)]))
    del g, stack
    return {"pattern": pattern, "steps": steps, "ms_per_step": ms,
            "tokens_per_s": wl.B * wl.Lq / (ms * 1e-3), "replay": "cuda graph"}


def decode_point(ic, dev, stream, flush, peaks, n_sms, clk):
    """decode_32k: B = 32 sequences, one new query each over a 32768-token
    cache, 16 layers (FSSS)x4 vs all-F; tokens/s = 32 tokens per step."""
    wl = synth.WORKLOADS["decode_32k"]
    layers = synth.make_layers(wl, indexer_for_all=True, device=dev)
    torch.cuda.synchronize()
    pt = {"config": {"B": wl.B, "Lq": wl.Lq, "Lk": wl.Lk, "q_offset": wl.q_offset,
                     "layers": wl.n_layers, "H_I": wl.H_I, "d_I": wl.d_I, "k": wl.k,
                     "Hq": wl.Hq, "d": wl.d}}
    for pat in (wl.pattern, "F" * wl.n_layers):
        key = "all_f" if pat == "F" * wl.n_layers else "fsss_x4"
        pt[key] = stack_point(ic, wl, pat, layers, stream, flush, peaks, n_sms, clk,
                              budget_ms=500.0, warmup=3)
    pt["speedup_of_pattern"] = pt["all_f"]["ms_per_step"] / pt["fsss_x4"]["ms_per_step"]
    pt["fsss_x4_graph"] = graph_point(ic, wl, wl.pattern, layers, flush)
    pt["all_f_graph"] = graph_point(ic, wl, "F" * wl.n_layers, layers, flush)
    pt["speedup_of_pattern_graph"] = (pt["all_f_graph"]["ms_per_step"]
                                      / pt["fsss_x4_graph"]["ms_per_step"])
    del layers
    torch.cuda.empty_cache()
    return pt


def e2e_leg(ic, stack, layers, pattern, stream, steps: int, pg, dev, tokens: float):
    """The same stack end to end through the public call with host buffers.
    Every step copies that step's inputs (every layer's q/K/V and the F
    layers' q_I/k_I/w) from pinned host memory to the device, runs the stack,
    and copies every layer's output back to pinned host memory; all of it is
    inside the timed region.  Steps are pipelined the way a serving loop
    would run them: two device copies of the inputs and outputs alternate, the
    host-to-device copies of step s+1 run on one copy stream and the
    device-to-host copies of step s-1 on another while step s computes.  The
    host copies are made once from the device-drawn inputs (drawing several
    GB on the host would take minutes)."""
    used = [{k: v for k, v in L.items() if k in ("q", "k", "v") or pattern[i] in "F1"}
            for i, L in enumerate(layers)]
    pinned = []
    for L in used:
        d = {}
        for k, v in L.items():
            h = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
            h.copy_(v)
            d[k] = h
        pinned.append(d)
    outs_host = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in stack.outs]
    h2d = sum(v.numel() * v.element_size() for L in pinned for v in L.values())
    d2h = sum(o.numel() * o.element_size() for o in stack.outs)

    # a second device copy of the inputs, and a second stack (its own outputs,
    # the first stack's workspace: both run on the compute stream, in order)
    layers2 = [{k: torch.empty_like(v) for k, v in L.items()} for L in layers]
    stack2 = ic.LayerStack(pattern, layers2, stack.dims, ws_bytes=16,
                           fused_topk=None if stack.opts is None else stack.opts.fused_topk,
                           z=0.0 if stack.opts is None else stack.opts.z)
    stack2.ws = stack.ws
    sets = [(layers, stack), (layers2, stack2)]
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    uploaded = [torch.cuda.Event() for _ in sets]
    computed = [torch.cuda.Event() for _ in sets]
    fetched = [torch.cuda.Event() for _ in sets]

    def upload(b):
        # set b's inputs are free once its last stack run is done
        up.wait_event(computed[b])
        with torch.cuda.stream(up):
            for i, L in enumerate(pinned):
                for k, v in L.items():
                    sets[b][0][i][k].copy_(v, non_blocking=True)
        uploaded[b].record(up)

    def run(b):
        stream.wait_event(uploaded[b])
        stream.wait_event(fetched[b])          # set b's outputs were read back
        sets[b][1].forward(stream)
        computed[b].record(stream)
        down.wait_event(computed[b])
        with torch.cuda.stream(down):
            for o, h in zip(sets[b][1].outs, outs_host):
                h.copy_(o, non_blocking=True)
        fetched[b].record(down)

    for b in range(2):                        # untimed warm-up of both sets
        computed[b].record(stream)
        fetched[b].record(down)
    for b in range(2):
        upload(b)
        run(b)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    t0.record(up)
    upload(0)
    for s in range(steps):
        b = s % 2
        if s + 1 < steps:
            upload(1 - b)                     # next step's inputs while this one computes
        run(b)
    end = torch.cuda.Event(enable_timing=True)
    end.record(down)
    up.wait_event(end)
    t1.record(up)
    torch.cuda.synchronize()
    e_ms, _, e_val = aggregate_over_ranks(t0.elapsed_time(t1) / steps, tokens, pg, dev)
    del pinned, outs_host, layers2, stack2
    return {"value": e_val, "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": e_ms, "steps": steps,
            "note": ("pinned host buffers; per step the inputs are copied in and every output "
                     "copied out; copies of neighbouring steps overlap the stack on two copy "
                     "streams (two device sets of inputs and outputs alternate)")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0,
                    help="timed steps (0: enough for a timed region of about 2 s, at least 20; "
                         "20 for the reference arm and the row-sharded mode)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill_64k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--pattern", default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-all-f", action="store_true")
    ap.add_argument("--fused-topk", type=int, default=-1, choices=[-1, 0, 1],
                    help="F layers: -1 the library's choice, 0 scores stored then top-k, "
                         "1 fused indexer -> top-k")
    ap.add_argument("--no-fused-compare", action="store_true",
                    help="skip timing the plain (unfused) top-k path beside the fused one")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the supplementary points (16-layer sweep, decode_32k)")
    ap.add_argument("--sweep", default="4,16,64,128",
                    help="sweep lengths in K tokens for the 16-layer all-F vs (FSSS)x4 points")
    ap.add_argument("--ref-rows", type=int, default=0,
                    help="query rows per step of the reference arm (0: 64, or 32 above 16K "
                         "tokens, where one row costs the oracle about 0.5 core-seconds)")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--shard", default="replicas", choices=["replicas", "rows"],
                    help="with N > 1 ranks: a replica of the workload per rank (weak scaling) "
                         "or one workload's query rows split over the ranks (strong scaling)")
    ap.add_argument("--rows-per-chunk", type=int, default=0,
                    help="F-layer score rows per chunk (0: as many as 16 GiB of scores allow)")
    args = ap.parse_args()
    wl = synth.WORKLOADS[args.workload]
    pattern = args.pattern or wl.pattern
    if len(pattern) != wl.n_layers:
        import dataclasses
        wl = dataclasses.replace(wl, n_layers=len(pattern), pattern=pattern)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    auto = args.steps <= 0
    if auto and (args.impl == "reference" or args.shard == "rows"):
        args.steps = 20
    if args.impl == "reference":
        return run_reference(args, wl, pattern)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    from lightning_indexer_top_relu_b200 import indexcache as ic

    if args.shard == "rows":
        return run_row_sharded(args, wl, pattern, ic, dev, world, rank, local, pg)

    peaks = load_peaks()
    need_all = (not args.no_all_f) and any(c in "S0" for c in pattern)
    layers = synth.make_layers(wl, indexer_for_all=need_all, device=dev)
    torch.cuda.synchronize()
    dims = ic.make_dims(wl.B, wl.Lq, wl.Lk, wl.q_offset, wl.H_I, wl.d_I, wl.Hq, wl.d, wl.k)
    rpc = args.rows_per_chunk if args.rows_per_chunk > 0 else default_rows_per_chunk(wl)
    fmode = None if args.fused_topk < 0 else args.fused_topk
    stack = ic.LayerStack(pattern, layers, dims, rows_per_chunk=rpc, fused_topk=fmode)
    lq_d = ic.layer_stack_dense_rows(dims, stack.ws.numel())
    stream = torch.cuda.current_stream()
    n = wl.n_layers
    npl = ic.MARKS_PER_LAYER
    flush = torch.empty(256 * 1024 * 1024 // 4, device=dev, dtype=torch.float32)
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count

    for _ in range(args.warmup):
        stack.forward(stream)
    torch.cuda.synchronize()
    if ic.get_last_device_error() != 0:
        raise RuntimeError("device error during warm-up")
    if auto:
        # one untimed probe step sizes the timed region (every rank takes the
        # slowest rank's figure, so all time the same number of steps)
        probe, _ = time_stack(ic, stack, stream, flush, 1, 0, with_marks=False)
        pms = torch.tensor([probe[0]], device=dev, dtype=torch.float64)
        if pg is not None:
            pg.all_reduce(pms, op=pg.ReduceOp.MAX)
        args.steps = timed_steps_for(float(pms.item()))

    marks = [new_marks(stream, n, npl) for _ in range(args.steps)]
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    clocks.start()
    launches0 = ic.kernel_launch_count()
    wall0 = time.perf_counter()
    for s in range(args.steps):
        flush.fill_(float(s))                    # L2 flush outside the step's events
        starts[s].record(stream)
        stack.forward(stream, events=marks[s][1])
        ends[s].record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    gpu_launches = ic.kernel_launch_count() - launches0
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    if ic.get_last_device_error() != 0:
        raise RuntimeError("device error during the timed steps")

    step_ms = [starts[s].elapsed_time(ends[s]) for s in range(args.steps)]
    local_ms = float(np.sum(step_ms)) / args.steps
    ms_per_step, tokens, value = aggregate_over_ranks(local_ms, float(wl.B * wl.Lq), pg, dev)

    w = work_per_layer(wl, lq_d)
    fused, fallback = fused_state(ic, stack)
    ki = kernel_times(wl, pattern, marks, args.steps, npl, w)
    sm_mhz = (clk or {}).get("sm_mhz") or 1965.0
    kernels, per_step = kernel_breakdown(ki, w, args.steps, ms_per_step, peaks, sm_mhz, n_sms,
                                         fused)
    roof = roofline_of(kernels, w, peaks, clk, wl.name)
    del marks

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Gaussian, correlated layers)",
            "config": config_of(wl, pattern, args), "gpu_launches": int(gpu_launches),
            "kernels": kernels, "roofline": roof,
            "indexer_share": (per_step.get("indexer", 0) + per_step.get("topk", 0)) / ms_per_step,
            "wall_s_timed": wall}
    if clk is not None:
        line["clocks"] = clk

    # ---- the fused indexer -> top-k against the plain path (scores stored per chunk)
    if fused:
        f_ms = float(np.mean(ki["indexer"])) + float(np.mean(ki["topk"]))
        ent = {"ms_per_f_layer": f_ms,
               "bytes_per_f_layer": w["fused_bytes"],
               "gbs": w["fused_bytes"] / (f_ms * 1e-3) / 1e9,
               "note": ("indexer + top-k of one F layer: inputs read once and index rows "
                        "written, no score stored; bound by the tensor cores, not by these bytes"),
               "fallback_blocks_last_f_layer": fallback}
        ent["frac_of_hbm"] = ent["gbs"] / peaks["hbm_gbs"]
        line["fused_topk"] = ent
    if fused and not args.no_fused_compare:
        ent = line["fused_topk"]
        f_ms = ent["ms_per_f_layer"]
        plain = ic.LayerStack(pattern, layers, dims, rows_per_chunk=rpc, fused_topk=0)
        ms_p, marks_p = time_stack(ic, plain, stream, flush, max(3, args.steps // 4), 1)
        ki_p = kernel_times(wl, pattern, marks_p, len(ms_p), npl, w)
        ent["plain_ms_per_f_layer"] = (float(np.mean(ki_p["indexer"]))
                                       + float(np.mean(ki_p["topk"])))
        ent["plain_ms_per_step"] = float(np.mean(ms_p))
        ent["speedup_of_fusion_per_f_layer"] = ent["plain_ms_per_f_layer"] / f_ms
        line["fused_topk"] = ent
        del plain, marks_p
        if ic.get_last_device_error() != 0:
            raise RuntimeError("device error in the plain-path leg")

    # ---- the same stack with every layer Full, for the F/S speed-up
    if need_all:
        stack_f = ic.LayerStack("F" * n, layers, dims, rows_per_chunk=rpc, fused_topk=fmode)
        k_f = max(3, args.steps // 2)
        ms_f, marks_f = time_stack(ic, stack_f, stream, flush, k_f, 2)
        msf = float(np.mean(ms_f))
        ki_f = kernel_times(wl, "F" * n, marks_f, k_f, npl, w)
        share_f = sum(float(np.sum(ki_f.get(k, [0.0]))) for k in ("indexer", "topk")) / k_f / msf
        msf, _, vf = aggregate_over_ranks(msf, float(wl.B * wl.Lq), pg, dev)
        line["all_f"] = {"pattern": "F" * n, "ms_per_step": msf, "value": vf, "steps": k_f,
                         "indexer_share": share_f, "speedup_of_pattern": msf / ms_per_step}
        del stack_f, marks_f
        line["cross_layer_overlap"] = cross_layer_overlap(ic, wl, layers, dims, rpc, stream,
                                                          peaks, n)
        if ic.get_last_device_error() != 0:
            raise RuntimeError("device error in the all-F leg")

    # ---- end to end through the public API with host buffers
    if not args.no_e2e:
        line["e2e"] = e2e_leg(ic, stack, layers, pattern, stream, max(3, min(args.steps, 300)), pg,
                              dev, float(wl.B * wl.Lq))
        if ic.get_last_device_error() != 0:
            raise RuntimeError("device error in the end-to-end leg")

    # ---- CPU oracle baseline (rank 0, N=1 only)
    if not args.no_cpu_baseline and world == 1:
        import oracle  # noqa: F401  (built and loaded before its timed sample)
        rps, sample, cores = oracle_rows_per_s(wl, pattern, layers, budget_s=args.cpu_budget_s)
        line["cpu_baseline"] = {"value": rps, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": sample}

    # ---- supplementary points (one GPU only): the 16-layer sweep and decode
    if not args.no_extras and world == 1:
        del stack, layers
        torch.cuda.empty_cache()
        lengths = [int(x) for x in args.sweep.split(",") if x.strip()]
        line["sweep_16_layers"] = sweep_points(ic, lengths, dev, stream, flush, peaks, n_sms, clk)
        line["decode_32k"] = decode_point(ic, dev, stream, flush, peaks, n_sms, clk)

    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
