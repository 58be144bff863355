"""bench.py's host-side bookkeeping (no GPU): the work model against closed
forms, the rule that ncu traffic is used only for the source it was captured
from, and input sizing."""
import os

import numpy as np
import pytest

import bench
from lightning_indexer_top_relu_b200 import synth


def test_work_model_closed_forms():
    wl = synth.custom(Lq=300, n_layers=1, H_I=4, d_I=64, k=100, Hq=16, d=128)
    w = bench.work_per_layer(wl, 0)
    sum_vis = 300 * 301 / 2                                    # rows t = 0..299 see t+1 keys
    sel = sum(min(t + 1, 100) for t in range(300))
    assert w["indexer_flops"] == 2 * 4 * 64 * sum_vis
    assert w["topk_bytes"] == 4 * sum_vis + 4 * 300 * 100
    assert w["gather_rows"] == 300 and w["dense_rows"] == 0
    assert w["gather_flops"] == 4 * 16 * 128 * sel
    assert w["gather_bytes"] == 4 * 128 * sel + 2 * 2 * 300 * 16 * 128 + 4 * 300 * 100


def test_work_model_splits_dense_and_gathered_rows():
    wl = synth.custom(Lq=300, n_layers=1, H_I=4, d_I=64, k=100, Hq=16, d=128)
    whole = bench.work_per_layer(wl, 0)
    split = bench.work_per_layer(wl, 296)                      # 37 blocks of 8 queries dense
    assert split["dense_rows"] == 296 and split["gather_rows"] == 4
    assert split["dense_flops"] + split["gather_flops"] == whole["gather_flops"]
    # block g (queries 8g..8g+7) runs ceil((8g+8)/64) tiles of 128 rows x 64 keys
    tiles = sum(-(-(8 * g + 8) // 64) for g in range(37))
    assert split["dense_tiles"] == tiles
    assert split["dense_exec_flops"] == tiles * 4 * 128 * 64 * 128
    assert split["dense_exec_exps"] == tiles * 128 * 64
    assert split["dense_exec_flops"] >= split["dense_flops"]


def test_profile_traffic_only_for_matching_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    csrc = tmp_path / "lightning_indexer_top_relu_b200" / "csrc"
    prof.mkdir()
    csrc.mkdir(parents=True)
    (csrc / "dense_attn.cuh").write_text("kernel v1")
    (csrc / "common.cuh").write_text("common")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    import hashlib
    h = hashlib.sha256(b"kernel v1" + b"common").hexdigest()[:16]
    (prof / "dense_attn_kernel_prefill_8k.md").write_text(
        f"source_hash: {h}\ndram_bytes_per_launch: 12345\n")
    assert bench.profile_traffic("dense_attn", "prefill_8k") == (12345, "dense_attn_kernel_prefill_8k.md")
    # no capture of this workload, and the one there is records no units: nothing to scale
    assert bench.profile_traffic("dense_attn", "prefill_64k", 65536) == (None, None)
    (csrc / "dense_attn.cuh").write_text("kernel v2")                      # source changed
    assert bench.profile_traffic("dense_attn", "prefill_8k") == (None, None)


def test_profile_traffic_scales_a_smaller_capture_by_its_rows(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    csrc = tmp_path / "lightning_indexer_top_relu_b200" / "csrc"
    prof.mkdir()
    csrc.mkdir(parents=True)
    (csrc / "sparse_attn.cuh").write_text("s")
    (csrc / "common.cuh").write_text("c")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    import hashlib
    h = hashlib.sha256(b"s" + b"c").hexdigest()[:16]
    (prof / "sparse_attn_kernel_layer_32k.md").write_text(
        f"source_hash: {h}\ndram_bytes_per_launch: 1000\nunits_per_launch: 16384\n")
    got, src = bench.profile_traffic("sparse_attn", "prefill_64k", 49152)
    assert got == 3000 and "sparse_attn_kernel_layer_32k.md" in src and "scaled" in src
    assert bench.profile_traffic("sparse_attn", "layer_32k", 16384)[0] == 1000
    (csrc / "sparse_attn.cuh").write_text("s2")                            # source changed
    assert bench.profile_traffic("sparse_attn", "prefill_64k", 49152) == (None, None)


def test_input_bytes_and_device_drawing_threshold():
    wl = synth.WORKLOADS["prefill_8k"]
    per_layer_attn = (8192 * 16 * 128 + 2 * 8192 * 128) * 2
    per_f_idx = 8192 * 32 * 128 * 2 + 8192 * 128 * 2 + 8192 * 32 * 4
    assert bench.input_bytes(wl, False) == 8 * per_layer_attn + 2 * per_f_idx
    assert bench.input_bytes(wl, True) == 8 * per_layer_attn + 8 * per_f_idx
    assert bench.input_bytes(wl, True) < 2 * 2 ** 30                       # drawn on the host
    assert bench.input_bytes(synth.WORKLOADS["prefill_64k"], True) > 2 * 2 ** 30


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _json_lines(out):
    import json
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def test_reference_arm_prints_one_line_with_its_baseline():
    """bench.py --impl reference: the oracle on host cores, W untimed
    warm-up steps, the same metric and config keys as the GPU arm, and
    cpu_baseline / e2e objects describing the run."""
    import subprocess
    import sys
    env = dict(os.environ, OMP_NUM_THREADS="1")      # what torchrun sets; must not shrink the pool
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                        "tiny_prefill", "--steps", "2", "--warmup", "1", "--ref-rows", "4"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    ln = lines[0]
    assert ln["impl"] == "reference" and ln["metric"] == bench.METRIC
    assert ln["unit"] == "tokens/s" and ln["higher_is_better"] is True and ln["value"] > 0
    assert ln["steps"] == 2 and ln["warmup"] == 1 and ln["n_gpus"] == 1
    assert ln["config"]["workload"] == "tiny_prefill"
    assert ln["cpu_baseline"]["kind"] == "oracle"
    assert ln["cpu_baseline"]["cores"] == bench.host_cores()
    assert ln["cpu_baseline"]["value"] == ln["value"]
    assert ln["e2e"] == {"value": ln["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                         "d2h_bytes_per_step": 0}


def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_under_two_ranks_prints_from_rank_0_only():
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                        "--master-port", str(_free_port()), "bench.py", "--impl", "reference", "--gpus",
                        "2", "--workload", "tiny_prefill", "--steps", "1", "--warmup", "1",
                        "--ref-rows", "2"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1 and lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2


def test_clock_sampler_reads_samples_through_a_pipe():
    """The sampler's parsing of nvidia-smi's CSV, fed by a stand-in command
    that prints three samples and then idles until it is stopped."""
    import sys
    import time
    rows = ["0, 1965, 1965, 512.3, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
            "0, 1950, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
            "0, 1980, 1965, 650.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"]
    script = ("import sys, time\n" + "".join(f"print({r!r}, flush=True)\n" for r in rows)
              + "time.sleep(60)\n")
    cs = bench.ClockSampler(0, cmd=[sys.executable, "-c", script])
    cs.start()
    time.sleep(1.0)
    out = cs.stop()
    assert out == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 3}
    missing = bench.ClockSampler(0, cmd=["/nonexistent/nvidia-smi"])
    missing.start()
    assert missing.stop() is None


@pytest.mark.parametrize("name,a1_tflop,a2_gb,a4_tflop,gather_gb", [
    ("prefill_8k", 0.275, 0.201, 0.120, 7.5),
    ("prefill_64k", 35.2, 9.1, 1.08, 67.7),
    ("sweep_128k", 140.7, 35.4, 2.18, 136.0),
    ("sweep_4k", 0.1375, None, 0.052, 3.2),
    ("sweep_16k", 2.20, None, 0.258, 16.1),
    ("decode_32k", 0.0172, 0.0045, 0.00054, 0.0335),
])
def test_work_model_matches_the_per_layer_work_table(name, a1_tflop, a2_gb, a4_tflop, gather_gb):
    """The roofline numerators against the per-layer algorithmic work
    tabulated for each configuration (indexer flops 2*H_I*d_I*sum(t+1), top-k
    bytes 4*sum(t+1) + 4*L*k, attention flops 4*Hq*d*V_k, logical K/V gather
    4*d*V_k; values rounded to about 3 digits)."""
    wl = synth.WORKLOADS[name]
    w = bench.work_per_layer(wl, 0)                      # every row counted as gathered
    t = np.arange(wl.Lq) + wl.q_offset
    vk = wl.B * np.minimum(np.minimum(t + 1, wl.Lk), wl.k).sum()

    def close(x, want):
        return abs(x - want) <= 0.015 * want
    assert close(w["indexer_flops"] / 1e12, a1_tflop)
    if a2_gb is not None:
        assert close(w["topk_bytes"] / 1e9, a2_gb)
    assert close(w["gather_flops"] / 1e12, a4_tflop)
    assert close(4.0 * wl.d * vk / 1e9, gather_gb)
    # the gather bytes add q, out and the index rows to the K/V rows
    extra = 2 * 2.0 * wl.B * wl.Lq * wl.Hq * wl.d + 4.0 * wl.B * wl.Lq * wl.k
    assert w["gather_bytes"] == pytest.approx(4.0 * wl.d * vk + extra)


def test_peaks_come_from_the_measured_file_else_the_fallback(tmp_path, monkeypatch):
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peaks()["source"] == "fallback"                     # no file
    f = tmp_path / "MEASURED_PEAKS.json"
    f.write_text("{not json")
    assert bench.load_peaks()["source"] == "fallback"
    f.write_text(json.dumps({"hbm_gbs": 6545.0}))                          # a key missing
    assert bench.load_peaks()["source"] == "fallback"
    f.write_text(json.dumps({"hbm_gbs": 6545.0, "bf16_tflops": 1652.8,
                             "bf16_tflops_sustained": 1386.2}))
    p = bench.load_peaks()
    assert p == {"hbm_gbs": 6545.0, "bf16_tflops": 1652.8, "bf16_tflops_sustained": 1386.2,
                 "source": "measured"}


def test_tensor_peak_is_sustained_only_when_the_power_cap_holds_clocks():
    peaks = {"hbm_gbs": 6459.9, "bf16_tflops": 1725.8, "bf16_tflops_sustained": 1391.2,
             "source": "measured"}
    assert bench.tensor_peak(peaks, None) == (1725.8, "burst")
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 20}
    assert bench.tensor_peak(peaks, full) == (1725.8, "burst")
    capped = dict(full, reasons=["sw_power_cap"], sm_mhz=1800.0)
    assert bench.tensor_peak(peaks, capped) == (1391.2, "sustained")
    slow = dict(full, sm_mhz=1700.0)
    assert bench.tensor_peak(peaks, slow) == (1391.2, "sustained")
    no_sus = dict(peaks, bf16_tflops_sustained=None)
    assert bench.tensor_peak(no_sus, capped) == (1725.8, "burst")


class _Ev:
    def __init__(self, t):
        self.t = t

    def elapsed_time(self, other):
        return other.t - self.t


def test_kernel_breakdown_and_roofline_from_stack_marks():
    """Two steps of a 2-layer FS stack with fake event times: the indexer,
    top-k and attention groups come from the right marks, shares add up,
    and the roofline names the largest share."""
    wl = synth.custom("fake", Lq=4096, n_layers=2, H_I=64, d_I=128, k=2048, Hq=16, d=128,
                      pattern="FS")
    w = bench.work_per_layer(wl, 0)
    npl = 5
    marks = []
    for s in range(2):
        # layer 0 F: indexer 3 ms, top-k 1 ms, attention 2 ms; layer 1 S: attention 2 ms
        t = [0, 3, 4, 4, 6, 6, 6, 6, 6, 8]
        marks.append(([_Ev(x) for x in t], None))
    ki = bench.kernel_times(wl, "FS", marks, 2, npl, w)
    assert ki["indexer"] == [3, 3] and ki["topk"] == [1, 1]
    assert ki["attn_gather"] == [2, 2, 2, 2] and "attn_dense" not in ki
    peaks = {"hbm_gbs": 6459.9, "bf16_tflops": 1725.8, "bf16_tflops_sustained": 1391.2,
             "source": "measured"}
    kern, per_step = bench.kernel_breakdown(ki, w, 2, 8.0, peaks, 1965.0, 148)
    assert abs(sum(k["share"] for k in kern.values()) - 1.0) < 1e-9
    assert kern["attn_gather"]["launches_per_step"] == 2
    assert abs(kern["indexer"]["tflops"] - w["indexer_flops"] / 3e-3 / 1e12) < 1e-6
    roof = bench.roofline_of(kern, w, peaks, None, "fake")
    assert roof["kernel"] == "sparse_attn" and roof["bound"] == "hbm"
    assert abs(roof["frac"] - roof["achieved"] / 6459.9) < 1e-12
    kern["indexer"]["share"] = 0.9
    roof = bench.roofline_of(kern, w, peaks, {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0,
                                              "reasons": ["sw_power_cap"]}, "fake")
    assert roof["kernel"] == "indexer_scores" and roof["peak_kind"] == "sustained"
    assert abs(roof["frac_of_burst"] - roof["achieved"] / 1725.8) < 1e-12


def test_default_workload_is_the_64k_prefill():
    import inspect
    src = inspect.getsource(bench.main)
    assert 'default="prefill_64k"' in src
    assert synth.WORKLOADS["prefill_64k"].pattern == "FSSSFSSS"


def test_uncorrelated_workloads_are_placed_on_the_requested_device():
    """The fixed-order draws of the tiny prefill land on the device asked for
    (the bench asks for the GPU); 'meta' stands in for it on the CPU."""
    layers = synth.make_layers(synth.WORKLOADS["tiny_prefill"], device="meta")
    assert len(layers) == 4
    assert all(t.device.type == "meta" for L in layers for t in L.values())
    host = synth.make_layers(synth.WORKLOADS["tiny_prefill"])
    assert all(t.device.type == "cpu" for L in host for t in L.values())


def test_timed_region_is_sized_to_about_two_seconds():
    assert bench.timed_steps_for(124.0) == 20          # the 64K step: 20 steps, 2.5 s
    assert bench.timed_steps_for(3.3) == 607           # the 8K step: about 2 s
    assert bench.timed_steps_for(0.12) == 2000         # capped
    assert bench.timed_steps_for(0.0) == 2000


def test_profile_traffic_scales_from_the_capture_nearest_in_size(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    csrc = tmp_path / "lightning_indexer_top_relu_b200" / "csrc"
    prof.mkdir()
    csrc.mkdir(parents=True)
    (csrc / "sparse_attn.cuh").write_text("s")
    (csrc / "common.cuh").write_text("c")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    import hashlib
    h = hashlib.sha256(b"s" + b"c").hexdigest()[:16]
    (prof / "sparse_attn_kernel_decode_32k.md").write_text(
        f"source_hash: {h}\ndram_bytes_per_launch: 32\nunits_per_launch: 32\n")
    (prof / "sparse_attn_kernel_layer_32k.md").write_text(
        f"source_hash: {h}\ndram_bytes_per_launch: 1000\nunits_per_launch: 16384\n")
    got, src = bench.profile_traffic("sparse_attn", "prefill_64k", 49152)
    assert got == 3000 and src.startswith("sparse_attn_kernel_layer_32k.md")
    got, src = bench.profile_traffic("sparse_attn", "decode_b64", 64)
    assert got == 64 and src.startswith("sparse_attn_kernel_decode_32k.md")
    # another regime (prefill rows from a decode capture) or a size more than
    # 4x away: no figure
    assert bench.profile_traffic("sparse_attn", "tiny_prefill", 32) == (None, None)
    assert bench.profile_traffic("sparse_attn", "prefill_512k", 16384 * 5) == (None, None)
    assert bench.profile_traffic("sparse_attn", "decode_b512", 512) == (None, None)
