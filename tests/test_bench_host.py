"""Host-side logic of bench.py that needs no GPU: the committed DRAM-traffic
record is used only while the kernel source still hashes to the captured one,
and the workload registry covers every configured workload."""
import hashlib
import json
import os

import bench
import synth


def _record(root, source_text, sha=None):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    src = os.path.join(root, "k.cu")
    with open(src, "w") as f:
        f.write(source_text)
    entry = {"kernel": "indexer_score", "config": {"workload": "w", "batch": 64}, "source": "k.cu",
             "source_sha256": sha or hashlib.sha256(source_text.encode()).hexdigest(),
             "bytes_per_launch": 1234}
    with open(os.path.join(root, "profiles", "dram_traffic.json"), "w") as f:
        json.dump({"entries": [entry]}, f)


def test_recorded_traffic_matches_source_hash(tmp_path):
    root = str(tmp_path)
    _record(root, "kernel v1")
    cfg = {"workload": "w", "batch": 64, "other": 1}
    assert bench.recorded_traffic("indexer_score", cfg, root=root) == 1234.0
    # another workload, another batch or another kernel: no record
    assert bench.recorded_traffic("indexer_score", {"workload": "x", "batch": 64}, root=root) is None
    assert bench.recorded_traffic("indexer_score", {"workload": "w", "batch": 32}, root=root) is None
    assert bench.recorded_traffic("attention", cfg, root=root) is None


def test_recorded_traffic_is_dropped_when_the_source_changed(tmp_path):
    root = str(tmp_path)
    _record(root, "kernel v2", sha=hashlib.sha256(b"kernel v1").hexdigest())
    assert bench.recorded_traffic("indexer_score", {"workload": "w", "batch": 64}, root=root) is None


def test_recorded_traffic_without_a_record(tmp_path):
    assert bench.recorded_traffic("indexer_score", {"workload": "w"}, root=str(tmp_path)) is None


def test_every_configured_workload_has_a_runner():
    assert set(bench.RUNNERS) == set(synth.WORKLOADS)
    assert bench.DEFAULT_WORKLOAD in bench.RUNNERS
    for name, (cls, cfg) in bench.RUNNERS.items():
        assert cfg.name == name and callable(getattr(cls, "step"))
