"""Host-side pieces of the bench's JSON line (no GPU): the DRAM traffic it
reports comes from the committed ncu capture only while the kernel sources
that capture ran are unchanged."""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

RECORDS = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))


@pytest.mark.parametrize("key", sorted(RECORDS))
def test_committed_traffic_records_match_the_current_sources(key):
    """Every committed capture still describes the kernels as they are, so the
    bench reports its traffic (a kernel edited since reads as null)."""
    rec = RECORDS[key]
    for src, want in rec["sources"].items():
        got = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()
        assert got == want, f"{src} changed since the {key} capture"
    assert bench.ncu_traffic(key) == rec["bytes_per_launch"] > 0


def test_traffic_is_null_once_a_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    sha = hashlib.sha256(src.read_bytes()).hexdigest()
    (prof / "ncu_traffic.json").write_text(json.dumps(
        {"k": {"sources": {"k.cu": sha}, "bytes_per_launch": 1234}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("k") == 1234
    assert bench.ncu_traffic("missing") is None
    src.write_text("kernel v2\n")
    assert bench.ncu_traffic("k") is None
    src.unlink()
    assert bench.ncu_traffic("k") is None
