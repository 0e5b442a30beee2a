"""bench.py's roofline arithmetic and bookkeeping, on CPU.

The algorithmic bytes and FLOPs are pinned to figures derived independently from the
model's shapes (the pi0.5 expert: 18 layers of 17,301,504 parameters plus action in/out;
the prefix pass: 17 full Gemma-2B-shaped layers plus one K/V-only layer at 544 tokens).
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_weight_bytes_per_step_are_the_expert_parameters():
    wl = bench.workload(1, "2-view")
    _, _, w_bytes_loop = bench.algorithmic(wl)
    params = 18 * 17_301_504 + 2 * 1024 * 32
    assert w_bytes_loop == params * 2 * 10
    assert abs(w_bytes_loop / 10 / 1e6 - 622.99) < 0.01


@pytest.mark.parametrize("name,batch,gb,tflop", [
    ("2-view", 1, 6.358, 0.4459),
    ("1-view", 1, 6.311, 0.3360),
    ("3-view", 4, 6.915, 1.886),
    ("3-view", 64, 17.055, 30.195),
])
def test_loop_bytes_and_flops(name, batch, gb, tflop):
    b, f, _ = bench.algorithmic(bench.workload(batch, name))
    assert abs(b / 1e9 - gb) < 0.002 and abs(f / 1e12 - tflop) < 0.002 * max(1.0, tflop)


def test_prefill_bytes_and_flops():
    b, f = bench.prefill_algorithmic(bench.workload(1, "e2e"))
    assert abs(f / 1e12 - 2.0788) < 1e-3
    assert abs(b / 1e9 - 3.7555) < 1e-3


def test_the_config_names_the_workload_only():
    c = bench.workload_config(bench.workload(1, "2-view"), 1)
    assert c["workload"] == "2-view L18 P512 Lv512 C63 B1"
    assert "engine" not in c and "l2" not in c


def test_traffic_is_reported_only_for_unchanged_kernel_sources(monkeypatch):
    name = "2-view L18 P512 Lv512 C63 B1"
    got = bench.measured_traffic(name, "persistent")
    assert got is None or got > 6e9          # the committed capture, when its hash matches
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 64)
    assert bench.measured_traffic(name, "persistent") is None
    assert bench.measured_traffic(name, "layered") is None


def test_vision_bytes_and_flops():
    # the SigLIP-So400m/14 matrices: patch 3*14*14 -> 1152, 27 x (q, k, v, o: 1152^2 each; fc1,
    # fc2: 1152 x 4304 each), projector 1152 -> 2048
    from synth import workloads as WL
    mats = 588 * 1152 + 27 * (4 * 1152 ** 2 + 2 * 1152 * 4304) + 2048 * 1152
    assert mats == 414_107_136
    b, f = bench.vision_algorithmic(WL.VisionShape(), 2)
    assert b == mats * 2 + 2 * 3 * 224 * 224 * 4 + 512 * 2048 * 2
    assert f == 2 * 512 * mats + 27 * 2 * 16 * 4 * 256 * 256 * 72
    assert abs(f / 1e9 - 440.35) < 0.01


def test_prefill_kernel_count_matches_the_launch_list():
    # 544-token prefill, 18 layers: 158 launches in the ncu launch list
    assert bench.prefill_kernels(18) == 158


def test_vision_reference_arm_prints_the_arms_metric_and_config(monkeypatch, capsys):
    import functools
    import json
    from types import SimpleNamespace

    from synth import workloads as WL
    monkeypatch.setattr(WL, "VisionShape", functools.partial(WL.VisionShape, n_layers=1))   # a short tower
    args = SimpleNamespace(workload="vision", views=2, steps=1, warmup=0, gpus=1, batch=1)
    bench.run_reference(args, 0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.vision_metric(2)
    assert line["config"] == bench.vision_config(WL.VisionShape(), 2, 1)
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
