"""Host logic of bench.py that needs no GPU: the DRAM-traffic lookup behind
roofline.traffic, and the throughput arithmetic of the JSON line.

The traffic lookup must report a capture only while the kernel source still has
the hash the capture was taken with, and only for the workload (name and head
count) it covers; otherwise the bench line carries traffic = null.
"""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import CONFIGS  # noqa: E402


def _fake_root(tmp_path, src_text, recorded_sha, workload="sol_sinks", heads=40, nbytes=1.5e9):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_text(src_text)
    rec = {"captures": [{"kernel": "attn_kernel<128>", "workload": workload, "heads_full": heads,
                         "source": "k.cu", "source_sha256": recorded_sha,
                         "dram_bytes_per_launch": nbytes}]}
    (tmp_path / "profiles" / "attn_traffic.json").write_text(json.dumps(rec))
    return str(tmp_path)


def test_traffic_reported_while_the_source_is_unchanged(tmp_path, monkeypatch):
    src = "kernel source\n"
    root = _fake_root(tmp_path, src, hashlib.sha256(src.encode()).hexdigest())
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.attn_traffic(CONFIGS["sol_sinks"]) == pytest.approx(1.5e9)


def test_traffic_dropped_once_the_source_changed(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, "edited kernel source\n", hashlib.sha256(b"kernel source\n").hexdigest())
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.attn_traffic(CONFIGS["sol_sinks"]) is None


def test_traffic_only_for_the_captured_workload(tmp_path, monkeypatch):
    src = "kernel source\n"
    sha = hashlib.sha256(src.encode()).hexdigest()
    root = _fake_root(tmp_path, src, sha, workload="long")
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.attn_traffic(CONFIGS["sol_sinks"]) is None
    assert bench.attn_traffic(CONFIGS["long"]) == pytest.approx(1.5e9)
    # a run on fewer heads than the capture was scaled to is another workload
    assert bench.attn_traffic(CONFIGS["long"].replace(H=4)) is None


def test_traffic_absent_without_a_record(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.attn_traffic(CONFIGS["sol_sinks"]) is None


def test_committed_record_is_well_formed():
    recs = json.load(open(os.path.join(ROOT, "profiles", "attn_traffic.json")))
    for rec in recs["captures"]:
        assert rec["workload"] in CONFIGS
        assert os.path.exists(os.path.join(ROOT, rec["source"]))
        assert os.path.exists(os.path.join(ROOT, rec["summary"]))
        assert rec["dram_bytes_per_launch"] == pytest.approx(
            rec["dram_bytes_per_launch_captured"] * rec["scale_to_full_launch"])
        assert rec["heads_full"] == CONFIGS[rec["workload"]].H
        assert rec["heads_full"] == rec["heads_captured"] * rec["scale_to_full_launch"]


def test_dense_equivalent_flops_of_the_default_workload():
    w = CONFIGS["sol_sinks"]
    # 4 B H N^2 d: S and P V over every (query, key) pair
    assert bench.dense_equiv_flops(w) == pytest.approx(4.0 * w.B * w.H * w.N * w.N * w.d)
    # whole-job throughput scales with the ranks at a fixed per-rank time
    assert bench.job_throughput(w, 2, 10.0) == pytest.approx(2 * bench.job_throughput(w, 1, 10.0))
