"""The committed DRAM-traffic records that bench.py's roofline objects carry (CPU only).

Each record in profiles/roofline_traffic.json names the kernel and workload, the command of
the ncu capture it came from, and the hashes of the sources the kernel was built from;
bench.py reports a record only while those hashes match. These checks keep the file
well-formed and its figures consistent with themselves.
"""
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
RECORDS = os.path.join(ROOT, "profiles", "roofline_traffic.json")


def _records():
    with open(RECORDS) as f:
        return json.load(f)["records"]


def test_records_are_well_formed():
    recs = _records()
    assert recs
    for rec in recs:
        for key in ("kernel", "workload", "dram_bytes_per_launch", "dram_read_bytes", "dram_write_bytes",
                    "launches_averaged", "sources_sha256", "command", "note"):
            assert key in rec, (rec.get("kernel"), key)
        assert "--clock-control none" in rec["command"]
        assert rec["dram_bytes_per_launch"] > 0
        assert abs(rec["dram_read_bytes"] + rec["dram_write_bytes"] - rec["dram_bytes_per_launch"]) <= 2
        for rel in rec["sources_sha256"]:
            assert os.path.exists(os.path.join(ROOT, rel)), rel


def test_per_launch_figures_average_to_the_record():
    for rec in _records():
        per = rec.get("per_launch")
        if not per:
            continue
        assert len(per) == rec["launches_averaged"]
        total = sum(p["dram_read_bytes"] + p["dram_write_bytes"] for p in per)
        assert abs(total / len(per) - rec["dram_bytes_per_launch"]) <= 1


def test_bench_reads_a_record_only_for_matching_sources(tmp_path, monkeypatch):
    rec = _records()[0]
    assert bench.recorded_traffic(rec["kernel"], "no such workload") is None
    # a copy of the tree whose first listed source differs: the record no longer applies
    first = next(iter(rec["sources_sha256"]))
    for rel in rec["sources_sha256"]:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        with open(os.path.join(ROOT, rel), "rb") as f:
            data = f.read()
        dst.write_bytes(data + (b"\n" if rel == first else b""))
    (tmp_path / "profiles").mkdir(exist_ok=True)
    (tmp_path / "profiles" / "roofline_traffic.json").write_text(open(RECORDS).read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic(rec["kernel"], rec["workload"]) is None
