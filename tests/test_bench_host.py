"""Host-side pieces of bench.py that need no GPU: the key that ties the committed
DRAM-traffic capture to the kernel sources it was taken on."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_source_key_ignores_comments_and_layout():
    code = "int f(int a) {\n    return a + 1;  // one more\n}\n"
    same = "/* doc */ int f(int a) { return a + 1; }"
    assert bench.source_code_tokens(code) == bench.source_code_tokens(same)


def test_source_key_sees_code_changes():
    assert bench.source_code_tokens("return a + 1;") != bench.source_code_tokens("return a + 2;")
    assert bench.source_code_tokens("x = y; // z") != bench.source_code_tokens("x = z; // y")



def test_traffic_figure_is_tied_to_its_sources(tmp_path, monkeypatch):
    """bench.py reports the committed traffic figure only for the sources it was
    taken on: a key that does not match gives None."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    entry = {"source_hash": bench.kernel_source_hash(), "bytes_per_launch_full_workload": 123.0}
    (prof / "traffic.json").write_text(json.dumps({"kda_chunk_fwd": entry}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: entry["source_hash"])
    assert bench.measured_traffic("kda_chunk_fwd") == 123.0
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "another")
    assert bench.measured_traffic("kda_chunk_fwd") is None
