"""Host logic of bench.py that needs no GPU: the profiled-traffic gate and the whole-job arithmetic."""
import json
import os
import sys

import pytest

HERE = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, HERE)
import bench  # noqa: E402


def test_traffic_is_reported_only_for_the_profiled_source(tmp_path, monkeypatch):
    rec = tmp_path / "profile.json"
    monkeypatch.setattr(bench, "PROFILE_JSON", str(rec))
    rec.write_text(json.dumps({"traffic_bytes_per_launch": 183014144, "csrc_sha256_16": bench.csrc_hash()}))
    assert bench.profiled_traffic() == 183014144.0
    rec.write_text(json.dumps({"traffic_bytes_per_launch": 183014144, "csrc_sha256_16": "0000000000000000"}))
    assert bench.profiled_traffic() is None  # the kernel source changed since the capture
    rec.write_text(json.dumps({"csrc_sha256_16": bench.csrc_hash()}))
    assert bench.profiled_traffic() is None  # no traffic figure
    rec.write_text("not json")
    assert bench.profiled_traffic() is None
    monkeypatch.setattr(bench, "PROFILE_JSON", str(tmp_path / "missing.json"))
    assert bench.profiled_traffic() is None


def test_source_hash_covers_every_profiled_file():
    h0 = bench.csrc_hash()
    assert len(h0) == 16 and int(h0, 16) >= 0
    for name in bench.PROFILED_SOURCES:
        assert os.path.isfile(os.path.join(HERE, "contextual_sparsity_ffn_b200", "csrc", name)), name


def test_whole_job_time_per_layer():
    # 4 ranks, 10 steps each, slowest rank 2 ms: 40 layer-steps in 2 ms
    assert bench.whole_job_us_per_layer(2.0, 10, 4) == pytest.approx(50.0)
    assert bench.whole_job_us_per_layer(2.0, 10, 1) == pytest.approx(200.0)
