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
    assert bench.profile_traffic("dense_attn", "prefill_8k") == 12345
    assert bench.profile_traffic("dense_attn", "prefill_64k") is None      # no capture
    (csrc / "dense_attn.cuh").write_text("kernel v2")                      # source changed
    assert bench.profile_traffic("dense_attn", "prefill_8k") is None


def test_input_bytes_and_device_drawing_threshold():
    wl = synth.WORKLOADS["prefill_8k"]
    per_layer_attn = (8192 * 16 * 128 + 2 * 8192 * 128) * 2
    per_f_idx = 8192 * 32 * 128 * 2 + 8192 * 128 * 2 + 8192 * 32 * 4
    assert bench.input_bytes(wl, False) == 8 * per_layer_attn + 2 * per_f_idx
    assert bench.input_bytes(wl, True) == 8 * per_layer_attn + 8 * per_f_idx
    assert bench.input_bytes(wl, True) < 2 * 2 ** 30                       # drawn on the host
    assert bench.input_bytes(synth.WORKLOADS["prefill_64k"], True) > 2 * 2 ** 30
