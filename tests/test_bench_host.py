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


def _random_csr(w, density, seed):
    import numpy as np
    rng = np.random.default_rng(seed)
    keep = rng.random((w.rows, w.nKB)) < density
    rp = np.zeros(w.rows + 1, np.int64)
    rp[1:] = np.cumsum(keep.sum(1))
    col = np.concatenate([np.nonzero(keep[r])[0] for r in range(w.rows)] + [np.zeros(0, np.int64)]).astype(np.int32)
    return keep, rp, col


def _issued_by_enumeration(w, keep, ecnt=None):
    """Tiles of the fine pass counted item by item (the docstring of issued_flops)."""
    import numpy as np
    per = 128 // w.q_block
    tiles = 0
    n_items = -(-w.N // 128)
    r0, r1 = w.dense_rows
    for bh in range(w.B * w.H):
        for it in range(n_items):
            if r1 > r0 and it * 128 >= r0 and min(it * 128 + 128, w.N) <= r1:
                continue
            u = np.zeros(w.nKB, bool)
            e = 0
            for qb in range(per * it, per * it + per):
                if qb < w.nQB:
                    u |= keep[bh * w.nQB + qb]
                    if ecnt is not None:
                        e += int(ecnt[bh * w.nQB + qb])
            tiles += (int(u.sum()) + 1) // 2
            if w.centroid:
                tiles += (-(-w.nKB // 64) + 1) // 2
            if ecnt is not None:
                tiles += (e + 127) // 128
    if r1 > r0:
        tiles += w.B * w.H * (-(-(r1 - r0) // 128)) * ((w.nKB + 1) // 2)
    return 4.0 * 128 * 128 * w.d * tiles


@pytest.mark.parametrize("case", ["sol_q64", "sla_q128", "sol_dense_extra"])
def test_issued_flops_count_every_tile(case):
    """issued_flops (the tensor-core work behind roofline.frac_issued) equals the
    tile-by-tile count on random kept-block masks: two query blocks per item for
    64-row blocks (union of their kept blocks), one for 128-row blocks, centroid
    and gathered tiles, dense rows and the items they replace."""
    import numpy as np
    import torch
    from workloads import Workload
    w = {
        "sol_q64": Workload("a", B=2, H=2, N=1300, d=64, dtype="bf16", method="sol", q_block=64, k_block=64),
        "sla_q128": Workload("b", B=1, H=3, N=2000, d=128, dtype="bf16", method="sla", q_block=128, k_block=64,
                             centroid=0),
        "sol_dense_extra": Workload("c", B=1, H=2, N=3000, d=128, dtype="bf16", method="sol", q_block=64,
                                    k_block=64, dense_rows=(200, 700), extra_tokens=64),
    }[case]
    keep, rp, col = _random_csr(w, 0.15, 7)
    ecnt = None
    if w.extra_tokens:
        ecnt = np.random.default_rng(8).integers(0, w.extra_tokens + 1, w.rows).astype(np.int32)
    got = bench.issued_flops(w, torch.from_numpy(rp), torch.from_numpy(col),
                             None if ecnt is None else torch.from_numpy(ecnt))
    assert got == _issued_by_enumeration(w, keep, ecnt)
    assert got >= bench.kept_flops(w, torch.from_numpy(rp), torch.from_numpy(col),
                                   None if ecnt is None else torch.from_numpy(ecnt)) * 0.999
