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


def test_scalar_gate_line_with_stand_in_device(monkeypatch):
    """The scalar-gate bench item's bookkeeping (bytes, throughput, keys), run with
    a stand-in for the library and the CUDA events."""
    import torch

    from gated_delta_rule_100_b200 import inputs, kda

    calls = []
    monkeypatch.setattr(kda, "gdn_chunk_fwd", lambda q, k, v, g, beta, scale, h0, **kw: calls.append(g.shape))
    monkeypatch.setattr(kda, "stream_status", lambda stream=None: kda.KDA_OK)

    class Event:
        def __init__(self, **kw):
            self.t = None

        def record(self, stream=None):
            self.t = len(calls)

        def elapsed_time(self, other):
            return 2.0 * (other.t - self.t)  # 2 ms per call

    monkeypatch.setattr(torch.cuda, "Event", Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)
    cfg = inputs.CONFIGS["oracle_scale_B1_H1_T256_d64"]
    d = inputs.make_config(cfg)
    P = {"hbm_gbs": 1000.0}
    r = bench.measure_scalar_gate(d, cfg, None, None, None, steps=4, warmup=2, P=P)
    assert calls == [(cfg.B, cfg.T, cfg.H)] * 6
    assert r["ms_per_step"] == 2.0 and r["value"] == cfg.B * cfg.T / 2e-3
    per_channel = bench.prefill_bytes(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.h0_std > 0, True)
    assert r["roofline"]["algorithmic_bytes_per_launch"] == per_channel - cfg.B * cfg.T * cfg.H * 4 * (cfg.dk - 1)
    assert r["entry_point"] == "kda_gdn_chunk_fwd"
