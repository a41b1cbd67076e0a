"""bench.py's host helpers: the DRAM-traffic figure is reported only for the
kernel source and workload it was measured on, and the HBM peak falls back to
the recipe's figure when no measured peaks file is present."""

import hashlib
import json
import os

import pytest

import bench


def kernel_sha():
    src = os.path.join(bench.ROOT, "moe_persistent_cta_b200", "csrc", "mk_kernel.cu")
    with open(src, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def test_traffic_scales_with_layers_for_the_measured_source(monkeypatch):
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {"kernel_sha256": kernel_sha(),
                                               "workload": "moe30b_b1",
                                               "fixed_bytes": 600e6, "per_layer_bytes": 100e6})
    assert bench.kernel_traffic("moe30b_b1", 48) == pytest.approx(600e6 + 48 * 100e6)
    assert bench.kernel_traffic("moe30b_b1", 2) == pytest.approx(800e6)


def test_traffic_is_null_for_another_source_or_workload(monkeypatch):
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {"kernel_sha256": "0" * 64,
                                               "workload": "moe30b_b1",
                                               "fixed_bytes": 600e6, "per_layer_bytes": 100e6})
    assert bench.kernel_traffic("moe30b_b1", 48) is None
    monkeypatch.setattr(bench, "NCU_TRAFFIC", dict(bench.NCU_TRAFFIC, kernel_sha256=kernel_sha()))
    assert bench.kernel_traffic("moe30b_b8_zipf", 48) is None


def test_recorded_traffic_is_close_to_the_algorithmic_bytes():
    """The committed figures describe a kernel that reads its bytes about once:
    per layer within 1 % of the 30B shape's algorithmic 113.8 MB."""
    t = bench.NCU_TRAFFIC
    assert abs(t["per_layer_bytes"] / 113.8e6 - 1.0) < 0.01
    assert 600e6 < t["fixed_bytes"] < 650e6


def test_hbm_peak_measured_and_fallback(tmp_path, monkeypatch):
    p = tmp_path / "peaks.json"
    p.write_text(json.dumps({"hbm_gbs": 6528.7}))
    monkeypatch.setattr(bench, "PEAKS_PATH", str(p))
    assert bench.hbm_peak() == (6528.7, "measured")
    monkeypatch.setattr(bench, "PEAKS_PATH", str(tmp_path / "missing.json"))
    assert bench.hbm_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    p.write_text("{not json")
    monkeypatch.setattr(bench, "PEAKS_PATH", str(p))
    assert bench.hbm_peak() == (bench.FALLBACK_HBM_GBS, "fallback")


def test_step_roofline_counts_the_touched_experts_and_the_kv():
    """The roofline's bytes are the active weights of the experts each layer
    touched plus the KV read, and frac = bytes / time / peak."""
    from moe_persistent_cta_b200 import configs
    shape = configs.MOE30B
    L = shape["n_layers"]
    r1 = bench.step_roofline(shape, [8192], [8] * L, 2.0)
    r8 = bench.step_roofline(shape, [8192], [16] * L, 2.0)
    expert = 3 * shape["d_ff"] * shape["d_model"] * 2
    assert r8["weight_bytes"] - r1["weight_bytes"] == L * 8 * expert
    kv_tok = L * 2 * shape["n_kv_heads"] * shape["head_dim"] * 2
    assert r1["kv_bytes"] == 8193 * kv_tok
    assert r1["bytes_per_step"] == r1["weight_bytes"] + r1["kv_bytes"]
    peak, _ = bench.hbm_peak()
    assert r1["achieved"] == pytest.approx(r1["bytes_per_step"] / 2e-3 / 1e9)
    assert r1["frac"] == pytest.approx(r1["achieved"] / peak)
    assert r1["experts_per_layer_mean"] == 8.0
    # the batch-1 30B step: about 6.08 GB, as the design notes state
    assert 6.0e9 < r1["bytes_per_step"] < 6.2e9
