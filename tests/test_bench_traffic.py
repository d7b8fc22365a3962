"""bench.py reports a kernel's DRAM traffic from an ncu capture only while the
kernel's source still hashes to the one captured: a changed kernel reports
null until it is captured again (no GPU needed)."""
import hashlib
import os

import bench


def test_recorded_traffic_matches_the_current_source():
    for (workload, kind), (nbytes, src, digest) in bench.MEASURED_TRAFFIC.items():
        with open(os.path.join(bench.ROOT, src), "rb") as f:
            assert hashlib.sha256(f.read()).hexdigest() == digest, (workload, kind, src)
        assert bench.measured_traffic(workload, kind) == nbytes


def test_unknown_kernel_reports_none():
    assert bench.measured_traffic("long32k", "no_such_kernel") is None
    assert bench.measured_traffic("no_such_workload", "lse_sweep") is None


def test_changed_source_reports_none(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cuh"
    src.write_bytes(b"// captured\n")
    digest = hashlib.sha256(b"// captured\n").hexdigest()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "MEASURED_TRAFFIC", {("w", "k"): (123.0, "kernel.cuh", digest)})
    assert bench.measured_traffic("w", "k") == 123.0
    src.write_bytes(b"// captured, then edited\n")
    assert bench.measured_traffic("w", "k") is None
    src.unlink()
    assert bench.measured_traffic("w", "k") is None
