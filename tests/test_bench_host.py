"""Host-side pieces of bench.py that need no GPU: the key that ties the committed
DRAM-traffic capture to the kernel sources it was taken on."""
import json
import os
import sys

import pytest

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
    """bench.py reports a committed traffic figure only while the kernel's device
    sources are those it was taken on: a key that does not match gives None."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    t = {"kernels": {"prep_kernel": {"source_hash": "abc", "captured_on": "w",
                                     "mean_bytes_per_launch": 123.0, "bytes_per_token_head": 7.0}}}
    (prof / "traffic.json").write_text(json.dumps(t))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kernel=None: "abc")
    assert bench.measured_traffic("prep_kernel") == (123.0, "w")
    assert bench.measured_traffic("prep_kernel", "bytes_per_token_head") == (7.0, "w")
    assert bench.measured_traffic("chain_kernel") == (None, None)
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kernel=None: "another")
    assert bench.measured_traffic("prep_kernel") == (None, None)


def test_kernel_source_keys_cover_their_files():
    """Each kernel's key changes with its own sources only."""
    assert bench.kernel_source_hash("prep_kernel") != bench.kernel_source_hash("chain_kernel")
    assert bench.kernel_source_hash("decode_step_kernel") != bench.kernel_source_hash()
    for files in bench.KERNEL_SOURCES.values():
        for name in files:
            assert os.path.exists(os.path.join(ROOT, "gated_delta_rule_100_b200", "csrc", name)), name


def test_record_traffic_from_ncu_csv(tmp_path):
    """The ncu CSV of prep, exact and chain launches on the long-context slice
    becomes per-kernel bytes per launch and per token-head, each keyed to that
    kernel's sources (an exact_prep_kernel launch is not taken for prep_kernel)."""
    import csv
    rows = [["ID", "Process ID", "Process Name", "Host Name", "Kernel Name", "Context", "Stream", "Block Size",
             "Grid Size", "Device", "CC", "Section Name", "Metric Name", "Metric Unit", "Metric Value"]]

    def add(i, kern, name, unit, val):
        rows.append([str(i), "1", "python", "h", kern, "1", "7", "(512,1,1)", "(296,1,1)", "0", "10.0", "",
                     name, unit, val])
    prep = "void prep_kernel<128, 0, 0>(CUtensorMap_st, CUtensorMap_st, PrepParams)"
    add(0, prep, "dram__bytes_read.sum", "Gbyte", "1.5")
    add(0, prep, "dram__bytes_write.sum", "Mbyte", "500")
    add(9, "void exact_prep_kernel<128, 0>(ExactParams)", "dram__bytes_read.sum", "byte", "24576")
    add(1, "void kda::chain_kernel<128, 64>(...)", "dram__bytes_read.sum", "Gbyte", "2.0")
    add(1, "void kda::chain_kernel<128, 64>(...)", "dram__bytes_write.sum", "byte", "1,000")
    add(2, prep, "dram__bytes_read.sum", "Gbyte", "1.0")
    add(2, prep, "dram__bytes_write.sum", "Gbyte", "1.0")
    path = tmp_path / "t.csv"
    with open(path, "w", newline="") as f:
        f.write("==PROF== Connected to process 1\n")
        csv.writer(f).writerows(rows)
    out = tmp_path / "traffic.json"
    t = bench.record_traffic(str(path), "long_context_slice_B1_H32_T65536_d128", str(out))
    p = t["kernels"]["prep_kernel"]
    assert p["source_hash"] == bench.kernel_source_hash("prep_kernel")
    assert p["launches_captured"] == 2 and p["bytes_per_launch"] == [2.0e9, 2.0e9]
    th = bench.prep_launch_token_heads(1, 65536, 32)
    assert th[:2] == [32 * 451 * 64] * 2 and sum(th) == 32 * 65536
    assert abs(p["bytes_per_token_head"] - 4.0e9 / (2 * 32 * 451 * 64)) < 1e-9
    assert t["kernels"]["chain_kernel"]["mean_bytes_per_launch"] == 2.0e9 + 1000
    assert t["kernels"]["exact_prep_kernel"]["launches_captured"] == 1


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


def _stand_in_events(monkeypatch, calls, ms_per_call=2.0):
    import torch

    class Event:
        def __init__(self, **kw):
            self.t = None

        def record(self, stream=None):
            self.t = len(calls)

        def elapsed_time(self, other):
            return ms_per_call * (other.t - self.t)

    monkeypatch.setattr(torch.cuda, "Event", Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: None)


def test_raw_prologue_line_with_stand_in_device(monkeypatch):
    """The raw-input item passes the workload's tensors as the raw projections with
    the workload's decay scale, and counts the per-channel prefill's bytes."""
    from gated_delta_rule_100_b200 import inputs, kda

    calls = []
    monkeypatch.setattr(kda, "chunk_fwd_raw", lambda q, k, v, g, beta, c, scale, h0, **kw: calls.append((g, c)))
    monkeypatch.setattr(kda, "stream_status", lambda stream=None: kda.KDA_OK)
    _stand_in_events(monkeypatch, calls)
    cfg = inputs.CONFIGS["oracle_scale_B1_H1_T256_d64"]
    d = inputs.make_config(cfg)
    r = bench.measure_raw(d, cfg, None, None, None, steps=3, warmup=1, P={"hbm_gbs": 1000.0})
    assert len(calls) == 4 and all(g is d["g"] and c == cfg.decay for g, c in calls)
    assert r["ms_per_step"] == 2.0 and r["entry_point"] == "kda_chunk_fwd_raw"
    assert r["roofline"]["algorithmic_bytes_per_launch"] == bench.prefill_bytes(
        cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.h0_std > 0, True)


def test_varlen_line_with_stand_in_device(monkeypatch):
    """The packed-batch item: the recipe's offsets reach the call, and the bytes are
    the tokens' plus one initial and one final state per sequence."""
    from gated_delta_rule_100_b200 import inputs, kda

    vc = inputs.VarlenConfig("tiny_varlen", 5, 2, 64, 64, 16, 300, 0.05, 0.02, 11)
    monkeypatch.setattr(inputs, "VARLEN_CONFIG", vc)
    calls = []

    def fake(q, k, v, g, beta, scale, cu, h0, **kw):
        calls.append(cu.tolist())
        assert q.shape[0] == cu[-1] and h0.shape == (vc.N, vc.H, vc.dk, vc.dv)

    monkeypatch.setattr(kda, "chunk_fwd_varlen", fake)
    monkeypatch.setattr(kda, "stream_status", lambda stream=None: kda.KDA_OK)
    _stand_in_events(monkeypatch, calls)
    r = bench.measure_varlen(None, steps=2, warmup=1, P={"hbm_gbs": 1000.0}, dev="cpu")
    lengths = inputs.varlen_lengths(vc)
    assert calls[0] == [0] + list(__import__("itertools").accumulate(lengths))
    assert all(vc.min_len <= n <= vc.max_len for n in lengths)
    T = sum(lengths)
    state = 4 * vc.dk * vc.dv * vc.N * vc.H
    assert r["config"]["T_total"] == T and r["value"] == T / 2e-3
    assert r["roofline"]["algorithmic_bytes_per_launch"] == bench.prefill_bytes(1, T, vc.H, vc.dk, vc.dv,
                                                                                False, False) + 2 * state


def test_two_level_line_restores_the_parts_hook(monkeypatch):
    """The few-heads item times the automatic choice, then the plain pass, and leaves
    the parts hook at automatic even when a call fails."""
    from gated_delta_rule_100_b200 import inputs, kda

    monkeypatch.setattr(inputs, "TWO_LEVEL_CONFIG", inputs.PrefillConfig("tiny", 1, 2, 256, 64, 64, 0.01, 0.02, 5))
    parts, calls = [], []
    monkeypatch.setattr(kda, "set_parts", lambda p: parts.append(p))
    monkeypatch.setattr(kda, "chunk_fwd", lambda *a, **kw: calls.append(parts[-1]))
    monkeypatch.setattr(kda, "stream_status", lambda stream=None: kda.KDA_OK)
    _stand_in_events(monkeypatch, calls)
    r = bench.measure_two_level(None, steps=2, warmup=1, P={"hbm_gbs": 1000.0}, dev="cpu")
    assert calls == [0, 0, 0, 1, 1, 1] and parts[-1] == 0
    assert r["ms_per_step"] == 2.0 and r["plain_pass_ms_per_step"] == 2.0

    def boom(*a, **kw):
        raise RuntimeError("device error")

    parts.clear()
    monkeypatch.setattr(kda, "chunk_fwd", boom)
    with pytest.raises(RuntimeError):
        bench.measure_two_level(None, steps=2, warmup=1, P={"hbm_gbs": 1000.0}, dev="cpu")
    assert parts[-1] == 0
