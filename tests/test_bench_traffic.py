"""The bench's `roofline.traffic` comes from an ncu capture recorded in
profiles/traffic.json with the SHA-256 of the captured kernel's sources: it is
reported only while those sources are unchanged (null once any of them
changes), and every workload that has an entry names existing source files."""
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _records():
    with open(bench.TRAFFIC_FILE) as f:
        return json.load(f)


def test_every_entry_is_a_workload_with_existing_sources():
    for name, rec in _records().items():
        assert name in bench.WORKLOADS, name
        assert rec["sources"], name
        for rel in rec["sources"]:
            assert os.path.exists(os.path.join(ROOT, rel)), (name, rel)
        assert rec["dram_bytes_per_launch"] > 0


def test_traffic_is_reported_for_unchanged_sources():
    for name, rec in _records().items():
        traffic, kernel = bench.captured_traffic(name)
        if rec["sources_sha256"] == bench.source_digest(rec["sources"]):
            assert traffic == float(rec["dram_bytes_per_launch"]) and kernel == rec["kernel"]
        else:
            assert traffic is None


def test_traffic_is_null_once_a_source_changes(tmp_path, monkeypatch):
    rec = _records()
    name = next(iter(rec))
    src = rec[name]["sources"][0]
    copy = tmp_path / "root"
    for rel in rec[name]["sources"]:
        (copy / os.path.dirname(rel)).mkdir(parents=True, exist_ok=True)
        with open(os.path.join(ROOT, rel), "rb") as f:
            (copy / rel).write_bytes(f.read())
    (copy / "profiles").mkdir()
    (copy / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(copy))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(copy / "profiles" / "traffic.json"))
    before, _ = bench.captured_traffic(name)
    with open(copy / src, "ab") as f:
        f.write(b"\n// edited\n")
    after, kernel = bench.captured_traffic(name)
    assert after is None and kernel == rec[name]["kernel"]
    assert before is None or before == float(rec[name]["dram_bytes_per_launch"])


def test_unknown_workload_has_no_traffic():
    assert bench.captured_traffic("no-such-workload") == (None, None)
