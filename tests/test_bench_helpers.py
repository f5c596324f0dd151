"""Host-side plumbing of bench.py (CPU only): the DRAM-traffic figure is
reported only while the kernel sources match the ones it was captured for."""
import hashlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture()
def bench(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench as b
    return b


def _sources_sha(b):
    h = hashlib.sha256()
    for f in b.KERNEL_SOURCES:
        with open(os.path.join(ROOT, "kv_cache_bit_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def test_traffic_reported_for_matching_sources(bench, tmp_path, monkeypatch):
    p = tmp_path / "traffic.md"
    p.write_text(f"x\ntraffic_bytes_per_call: 1234\nsource_sha256: {_sources_sha(bench)}\n")
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(p))
    assert bench.decode_traffic() == 1234.0


def test_traffic_withheld_after_a_source_change(bench, tmp_path, monkeypatch):
    p = tmp_path / "traffic.md"
    p.write_text("traffic_bytes_per_call: 1234\nsource_sha256: " + "0" * 64 + "\n")
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(p))
    assert bench.decode_traffic() is None


def test_traffic_withheld_without_a_profile(bench, tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(tmp_path / "missing.md"))
    assert bench.decode_traffic() is None
