#!/usr/bin/env python
"""Benchmark of the KDA forward path on B200: chunkwise prefill (the step) and
single-step decode, printed as one JSON line by rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Step: one kda_chunk_fwd over the long-context workload (B=1, H=32,
T=1,048,576, dk=dv=128; bf16 q/k/v, fp32 g and beta, zero h0, out bf16 +
final state fp32).  Inputs are synthetic (gated_delta_rule_100_b200.inputs),
resident in HBM before the timed region, and 51.7 GB per step (far above the
126 MB L2, so no flush is needed between steps).  Value: tokens (B*T) per
second over all ranks; each rank runs its own copy of the workload (weak
scaling, no collective on the data path).  Timing: CUDA events on the
launching stream, barrier + synchronize on both sides, max over ranks.

Also measured and reported in the same line:
  decode   64 consecutive kda_decode_step calls on B=256, H=32, d=128 with a
           512 MiB fp32 state (GB/s of algorithmic traffic);
  e2e      the same prefill metric through kda_chunk_fwd_host with pinned host
           buffers: H2D of the inputs, the kernels, D2H of out and hT per step
           (pieces of the token axis overlapped on three streams);
  roofline achieved algorithmic GB/s of the prefill call (its kernels) vs
           measured HBM peak, with each kernel's busy time from one extra step
           whose launches the kernels stamp themselves (%globaltimer);
  training the training-shape prefill (B8 H32 T4096) timed the same way;
  raw_prologue  kda_chunk_fwd_raw (gate prologue fused) on the step's workload;
  varlen   kda_chunk_fwd_varlen on a packed batch of 64 sequences of mixed lengths;
  two_level  a few-heads long sequence (B1 H4 T262144) with and without the
           two-level pass;
  backward kda_chunk_bwd on the training shape (fp32 CUDA cores, "alu" roofline);
  cpu_baseline  the fp64 oracle on a bounded sample of the workload (rank 0,
           N = 1 only), plus every workload's recipe on 1 thread and all cores.

--record-traffic CSV writes profiles/traffic.json from an ncu capture of the
DRAM-bytes counters (taken on --workload) and exits.

--impl reference times the fp64 oracle (the only reference that exists for
this method) on the host cores, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "long_context_B1_H32_T1M_d128"
METRIC = "KDA prefill tokens/s & TFLOP/s; decode-step state GB/s vs B200 HBM peak"
CHUNK = 64
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers ----
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def prefill_bytes(B, T, H, dk, dv, with_h0, with_hT):
    """Algorithmic HBM bytes of one prefill launch: q, k, v (bf16), g (fp32),
    beta (fp32) read once, out (bf16) written once, h0/hT (fp32) once."""
    per_token_head = 2 * dk * 2 + dv * 2 + 4 * dk + 4 + 2 * dv
    state = 4 * dk * dv * B * H
    return B * T * H * per_token_head + (state if with_h0 else 0) + (state if with_hT else 0)


def measure_scalar_gate(d, cfg, out, hT, stream, steps, warmup, P):
    """The scalar-gate (Gated DeltaNet) prefill on the bench workload: the same
    inputs with one log-decay per token and head (key channel 0 of the workload's
    gate), timed like the step.  Device-side inputs; one process's own timing."""
    import torch

    from gated_delta_rule_100_b200 import kda

    gs = d["g"][..., 0].contiguous()

    def step():
        kda.gdn_chunk_fwd(d["q"], d["k"], d["v"], gs, d["beta"], cfg.scale, d["h0"], out=out, hT=hT,
                          stream=stream)

    for _ in range(max(1, warmup)):
        step()
    torch.cuda.synchronize()
    if kda.stream_status(stream) != kda.KDA_OK:
        raise RuntimeError("device-side error during warm-up")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if kda.stream_status(stream) != kda.KDA_OK:
        raise RuntimeError("device-side error in the timed steps")
    ms = e0.elapsed_time(e1) / steps
    # the gate is 4 bytes per token-head instead of 4 dk
    nbytes = (prefill_bytes(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.h0_std > 0, True)
              - cfg.B * cfg.T * cfg.H * 4 * (cfg.dk - 1))
    achieved = nbytes / (ms / 1e3) / 1e9
    del gs
    return {"metric": "scalar-gate prefill tokens/s", "value": cfg.B * cfg.T / (ms / 1e3), "unit": "tokens/s",
            "ms_per_step": ms, "steps": steps, "entry_point": "kda_gdn_chunk_fwd",
            "config": {"workload": cfg.name, "gate": "fp32 [B,T,H]: key channel 0 of the workload's gate"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": P["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / P["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes}}


def _time_calls(step, stream, steps, warmup):
    """Mean ms of `steps` calls of `step` on `stream` after `warmup` untimed ones,
    CUDA events on the stream; raises if the library reports a device-side error."""
    import torch

    from gated_delta_rule_100_b200 import kda

    for _ in range(max(1, warmup)):
        step()
    torch.cuda.synchronize()
    if kda.stream_status(stream) != kda.KDA_OK:
        raise RuntimeError("device-side error during warm-up")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if kda.stream_status(stream) != kda.KDA_OK:
        raise RuntimeError("device-side error in the timed steps")
    return e0.elapsed_time(e1) / steps


def _hbm_roofline(nbytes, ms, P):
    achieved = nbytes / (ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": P["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / P["hbm_gbs"], "algorithmic_bytes_per_launch": nbytes}


def measure_raw(d, cfg, out, hT, stream, steps, warmup, P):
    """The fused gate prologue (kda_chunk_fwd_raw) on the bench workload: its
    tensors passed as the raw projections (q, k normalised again in the kernels,
    g = -c softplus(g_raw) with c = the workload's decay scale, beta = sigmoid of
    the workload's beta), timed like the step."""
    from gated_delta_rule_100_b200 import kda

    c = cfg.decay

    def step():
        kda.chunk_fwd_raw(d["q"], d["k"], d["v"], d["g"], d["beta"], c, cfg.scale, d["h0"], out=out, hT=hT,
                          stream=stream)

    ms = _time_calls(step, stream, steps, warmup)
    nbytes = prefill_bytes(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.h0_std > 0, True)
    return {"metric": "raw-input prefill tokens/s", "value": cfg.B * cfg.T / (ms / 1e3), "unit": "tokens/s",
            "ms_per_step": ms, "steps": steps, "entry_point": "kda_chunk_fwd_raw",
            "config": {"workload": cfg.name, "raw": "the workload's q, k, g, beta as raw projections",
                       "gate_c": c},
            "roofline": _hbm_roofline(nbytes, ms, P)}


def measure_varlen(stream, steps, warmup, P, dev):
    """A packed batch (kda_chunk_fwd_varlen): 64 sequences of log-uniform lengths in
    [128, 16384] (269,705 tokens), 32 heads, a state per sequence in and out."""
    import torch

    from gated_delta_rule_100_b200 import inputs, kda

    vc = inputs.VARLEN_CONFIG
    d = inputs.make_varlen(vc, device=dev)
    T = d["q"].shape[0]
    out = torch.empty((T, vc.H, vc.dv), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((vc.N, vc.H, vc.dk, vc.dv), dtype=torch.float32, device=dev)

    def step():
        kda.chunk_fwd_varlen(d["q"], d["k"], d["v"], d["g"], d["beta"], vc.scale, d["cu_seqlens"], d["h0"],
                             out=out, hT=hT, stream=stream)

    ms = _time_calls(step, stream, steps, warmup)
    state = 4 * vc.dk * vc.dv * vc.N * vc.H
    nbytes = prefill_bytes(1, T, vc.H, vc.dk, vc.dv, False, False) + 2 * state
    lengths = inputs.varlen_lengths(vc)
    del d, out, hT
    return {"metric": "packed-batch prefill tokens/s", "value": T / (ms / 1e3), "unit": "tokens/s",
            "ms_per_step": ms, "steps": steps, "entry_point": "kda_chunk_fwd_varlen",
            "config": {"workload": vc.name, "N": vc.N, "T_total": T, "H": vc.H, "dk": vc.dk, "dv": vc.dv,
                       "min_len": min(lengths), "max_len": max(lengths), "seed": vc.seed},
            "roofline": _hbm_roofline(nbytes, ms, P)}


def measure_two_level(stream, steps, warmup, P, dev):
    """Few heads, long sequence (B1 H4 T262144): kda_chunk_fwd with its automatic
    two-level pass, and the same call with the two-level pass off (one chain CTA
    per (b, h, value slice) walking all 4,096 chunks)."""
    import torch

    from gated_delta_rule_100_b200 import inputs, kda

    tc = inputs.TWO_LEVEL_CONFIG
    d = inputs.make_config(tc, device=dev)
    out = torch.empty((tc.B, tc.T, tc.H, tc.dv), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((tc.B, tc.H, tc.dk, tc.dv), dtype=torch.float32, device=dev)

    def step():
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], tc.scale, d["h0"], out=out, hT=hT, stream=stream)

    try:
        kda.set_parts(0)
        ms = _time_calls(step, stream, steps, warmup)
        kda.set_parts(1)
        ms_plain = _time_calls(step, stream, steps, warmup)
    finally:
        kda.set_parts(0)
    nbytes = prefill_bytes(tc.B, tc.T, tc.H, tc.dk, tc.dv, tc.h0_std > 0, True)
    del d, out, hT
    return {"metric": "few-heads long-sequence prefill tokens/s", "value": tc.B * tc.T / (ms / 1e3),
            "unit": "tokens/s", "ms_per_step": ms, "plain_pass_ms_per_step": ms_plain, "steps": steps,
            "entry_point": "kda_chunk_fwd (two-level pass chosen automatically)",
            "config": {"workload": tc.name, "B": tc.B, "H": tc.H, "T": tc.T, "dk": tc.dk, "dv": tc.dv},
            "roofline": _hbm_roofline(nbytes, ms, P)}


def prefill_flops(B, T, H, dk, dv, C=CHUNK):
    """Algorithmic flops of the chunkwise form (triangles counted once): the three
    state contractions, A, the triangular solve, the causal q k^T and P Vnew."""
    per = (6 * dk * dv + (C - 1) * dk + (C - 1) * (dk + dv) + (C + 1) * (dk + dv))
    return B * T * H * per


def decode_bytes(B, H, dk, dv):
    """State read + written (fp32) and q, k, v, g, beta, out per (b, h)."""
    return B * H * (2 * 4 * dk * dv + 2 * dk * 2 + dv * 2 + 4 * dk + 4 + 2 * dv)


def source_code_tokens(text):
    """C/C++/CUDA source with comments removed and whitespace runs collapsed, so a
    comment-only edit keeps the key of measurements taken on that code."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


# The device sources each captured kernel is built from (its file and the headers
# it includes): a traffic figure stays valid while these are unchanged.
COMMON_HEADERS = ("chunk_common.cuh", "chunk_params.cuh", "kda_device.cuh")
KERNEL_SOURCES = {
    "prep_kernel": ("prep_fwd.cu",) + COMMON_HEADERS,
    "exact_prep_kernel": ("exact_prep.cu",) + COMMON_HEADERS,
    "chain_kernel": ("chain_fwd.cu",) + COMMON_HEADERS,
    "decode_step_kernel": ("decode.cu", "kda_device.cuh"),
}


def kernel_source_hash(kernel=None):
    """sha256 (first 16 hex digits) of a kernel's device sources (all of csrc when
    kernel is None), comments removed and whitespace collapsed."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_100_b200", "csrc")
    names = sorted(KERNEL_SOURCES[kernel]) if kernel else sorted(
        n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh")))
    for name in names:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + source_code_tokens(f.read()).encode())
    return h.hexdigest()[:16]


REC_BYTES = 74240            # one chunk record of one (b, h)
RECORD_CAP = 2 << 30         # bytes of records the prefill workspace holds at once
TRAFFIC_KERNELS = ("prep_kernel", "chain_kernel", "exact_prep_kernel", "decode_step_kernel")


def prep_launch_token_heads(B, T, H):
    """Token-heads (and chunks) of each prep/chain launch of kda_chunk_fwd on
    [B, T, H] (the library's segmentation: all chunks when their records fit the
    cap, else segments of as many chunks as fit in half of it)."""
    nch = -(-T // CHUNK)
    row = B * H * REC_BYTES
    seg = nch if nch * row <= RECORD_CAP else max(1, RECORD_CAP // (2 * row))
    out = []
    for n0 in range(0, nch, seg):
        cnt = min(seg, nch - n0)
        out.append(B * H * min(cnt * CHUNK, T - n0 * CHUNK))
    return out


def record_traffic(csv_path, workload, out_path=None):
    """Turn an ncu --csv log of dram__bytes_read.sum / dram__bytes_write.sum
    (one or more kernels, each launch complete) into profiles/traffic.json, keyed
    to the current kernel sources.  Per kernel: the mean bytes per launch and, for
    the prefill kernels, per token-head of the captured launches (the launches are
    in issue order, so the n-th prep or chain launch is segment n)."""
    import csv

    from gated_delta_rule_100_b200 import inputs

    launches = {}  # launch id -> (kernel, bytes)
    order = []
    with open(csv_path) as f:
        rows = [r for r in csv.reader(f) if r and not r[0].startswith("==")]
    head = rows[0]
    idx = {k: head.index(k) for k in ("ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value")}
    scale_of = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}
    for r in rows[1:]:
        if r[idx["Metric Name"]] not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            continue
        lid = r[idx["ID"]]
        # the function's own name: "void ns::name<...>(args)" -> "name"
        base = r[idx["Kernel Name"]].split("(")[0].split("<")[0].split()[-1].split("::")[-1]
        name = base if base in TRAFFIC_KERNELS else None
        if name is None:
            continue
        val = float(r[idx["Metric Value"]].replace(",", "")) * scale_of.get(r[idx["Metric Unit"]], 1.0)
        if lid not in launches:
            launches[lid] = [name, 0.0]
            order.append(lid)
        launches[lid][1] += val
    cfg = inputs.CONFIGS.get(workload)
    per_launch_th = prep_launch_token_heads(cfg.B, cfg.T, cfg.H) if cfg is not None else []
    kernels = {}
    for name in TRAFFIC_KERNELS:
        ids = [i for i in order if launches[i][0] == name]
        if not ids:
            continue
        e = {"source_hash": kernel_source_hash(name), "launches_captured": len(ids),
             "bytes_per_launch": [launches[i][1] for i in ids]}
        e["mean_bytes_per_launch"] = sum(e["bytes_per_launch"]) / len(ids)
        if name in ("prep_kernel", "chain_kernel") and per_launch_th:
            th = [per_launch_th[n % len(per_launch_th)] for n in range(len(ids))]
            e["bytes_per_token_head"] = sum(e["bytes_per_launch"]) / sum(th)
        kernels[name] = e
    out_path = out_path or os.path.join(ROOT, "profiles", "traffic.json")
    t = {"kernels": {}}
    if os.path.exists(out_path):  # captures of other kernels stay
        with open(out_path) as f:
            t = json.load(f)
    for name, e in kernels.items():
        e["captured_on"] = workload
        t.setdefault("kernels", {})[name] = e
    t["source_key"] = ("per kernel: sha256 of its device sources (bench.KERNEL_SOURCES) with comments removed "
                       "and whitespace collapsed")
    with open(out_path, "w") as f:
        json.dump(t, f, indent=1)
    return t


def measured_traffic(kernel, field="mean_bytes_per_launch"):
    """A kernel's DRAM-traffic figure from profiles/traffic.json, if that capture
    was taken on the kernel's current device sources (else None), with the
    workload it was captured on."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None, None
    with open(path) as f:
        t = json.load(f)
    e = t.get("kernels", {}).get(kernel)
    if not e or field not in e or e.get("source_hash") != kernel_source_hash(kernel):
        return None, None
    return e[field], e.get("captured_on")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        time.sleep(0.2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""
        else:
            self.out = ""

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "gloo" if args.impl == "reference" else "nccl"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def weak_value(units_per_step, world, steps, total_ms):
    """Whole-job throughput: every rank processes its own units each step."""
    return units_per_step * world * steps / (total_ms / 1e3)


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------- cpu oracle ----
def oracle_rate(d, scale, heads, tokens, threads):
    """Run the fp64 oracle on `heads` x first `tokens` tokens; returns (seconds, token-heads)."""
    import oracle
    import torch

    def cut(t):
        return t[:, :tokens, :heads].to("cpu", torch.float64).numpy()

    args = [cut(d[k]) for k in ("q", "k", "v", "g", "beta")]
    t0 = time.perf_counter()
    oracle.kda_fwd(*args, scale, None, threads=threads)
    return time.perf_counter() - t0, heads * tokens * d["q"].shape[0]


def cpu_baseline(d, cfg, budget_s):
    """Oracle throughput on a bounded sample sized to about `budget_s` seconds."""
    cores = os.cpu_count() or 1
    heads = min(cfg.H, cores)
    dt, n = oracle_rate(d, cfg.scale, heads, 512, heads)
    rate = n / max(dt, 1e-9)
    tokens = int(min(cfg.T, max(512, rate * budget_s / heads)))
    tokens = max(512, (tokens // 512) * 512)
    dt, n = oracle_rate(d, cfg.scale, heads, tokens, heads)
    th_per_s = n / dt
    return {"value": th_per_s / cfg.H, "unit": "tokens/s", "cores": heads, "kind": "oracle",
            "sample": f"fp64 oracle on heads 0-{heads - 1} x first {tokens} tokens of the workload "
                      f"({n} token-heads, {dt:.1f} s, {heads} threads); tokens/s = token-heads/s / {cfg.H}"}


def measure_training(P, peak_src, stream, steps, warmup, dev):
    """The training-shape prefill (B8 H32 T4096 d128, 1.65 GB of inputs: above L2,
    no flush) through kda_chunk_fwd, timed like the step, with its own roofline."""
    import torch

    from gated_delta_rule_100_b200 import inputs, kda

    cfg = inputs.CONFIGS["training_B8_H32_T4096_d128"]
    d = inputs.make_config(cfg, device=dev)
    out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.dv), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((cfg.B, cfg.H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)

    def step():
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], cfg.scale, d["h0"], out=out, hT=hT,
                      stream=stream)

    for _ in range(max(3, warmup)):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if kda.stream_status(stream) != kda.KDA_OK:
        raise RuntimeError("device-side error in the training-shape steps")
    ms = e0.elapsed_time(e1) / steps
    kda.kernel_times()
    kda.kernel_timing(True)
    step()
    torch.cuda.synchronize()
    kda.kernel_timing(False)
    kt = kda.kernel_times()
    nbytes = prefill_bytes(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.h0_std > 0, True)
    nflops = prefill_flops(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv)
    achieved = nbytes / (ms / 1e3) / 1e9
    return {"metric": "training-shape prefill tokens/s", "value": cfg.B * cfg.T / (ms / 1e3), "unit": "tokens/s",
            "ms_per_step": ms, "steps": steps, "tflops": nflops / (ms / 1e3) / 1e12,
            "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "T": cfg.T, "dk": cfg.dk, "dv": cfg.dv,
                       "l2": "inputs 1.65 GB, larger than L2; no flush"},
            "kernels": {k: {"ms": t, "launches": n} for k, (t, n) in kt.items() if n > 0},
            "roofline": {"kernel": "kda_chunk_fwd (prep_kernel + chain_kernel)", "bound": "hbm",
                         "achieved": achieved, "peak": P["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / P["hbm_gbs"], "peak_source": peak_src,
                         "algorithmic_bytes_per_launch": nbytes,
                         "tensor_view": {"achieved_tflops": nflops / (ms / 1e3) / 1e12,
                                         "peak_tflops": P["bf16_tflops_sustained"],
                                         "frac": nflops / (ms / 1e3) / 1e12 / P["bf16_tflops_sustained"]}}}


# fp32 CUDA-core peak of the B200, from its unit counts and clock: 148 SMs x 128
# fp32 lanes x 2 flops (FMA) x the measured maximum SM clock.
def fp32_alu_peak_tflops(P):
    return 148 * 128 * 2 * P.get("sm_max_mhz", 1965.0) * 1e6 / 1e12


def backward_flops(B, T, H, dk, dv):
    """Algorithmic flops of the recurrence's backward, once per token: the
    forward step it differentiates (decay, p = S'^T k, the write: ~5 dk dv) and
    the reverse step (S', p, S_t, dq, dS += q do, du, dk (two terms), dS', dalpha,
    dS_{t-1}: ~20 dk dv).  Recomputation from checkpoints is not counted."""
    return B * T * H * 25 * dk * dv


def backward_bytes(B, T, H, dk, dv):
    """Algorithmic HBM bytes: q, k, v, dout (bf16), g, beta read; dq, dk, dv (bf16),
    dg, dbeta (fp32) written."""
    return B * T * H * (2 * (2 * dk + 2 * dv) + 4 * dk + 4 + 2 * (2 * dk + dv) + 4 * dk + 4)


def measure_backward(P, stream, steps, dev):
    """kda_chunk_bwd on the training shape with a random dL/dout, timed like the
    step (3 warm-ups), with its roofline: the recurrent form is bound by fp32
    CUDA-core arithmetic ("alu"), against the unit-count peak."""
    import torch

    from gated_delta_rule_100_b200 import inputs, kda

    cfg = inputs.CONFIGS["training_B8_H32_T4096_d128"]
    d = inputs.make_config(cfg, device=dev)
    gen = torch.Generator(device=dev).manual_seed(cfg.seed + 100)
    dout = torch.randn((cfg.B, cfg.T, cfg.H, cfg.dv), generator=gen, device=dev).to(torch.bfloat16)

    def step():
        return kda.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], cfg.scale, d["h0"], dout, None,
                             stream=stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(1, min(steps, 3))
    e0.record(stream)
    for _ in range(n):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if kda.stream_status(stream) != kda.KDA_OK:
        raise RuntimeError("device-side error in the backward steps")
    ms = e0.elapsed_time(e1) / n
    fl = backward_flops(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv)
    peak = fp32_alu_peak_tflops(P)
    return {"metric": "training-shape backward tokens/s", "value": cfg.B * cfg.T / (ms / 1e3), "unit": "tokens/s",
            "ms_per_step": ms, "steps": n, "entry_point": "kda_chunk_bwd",
            "config": {"workload": cfg.name, "cotangents": "dL/dout ~ N(0, 1) bf16, dL/dhT = 0"},
            "roofline": {"kernel": "kda_chunk_bwd (recurrent form: checkpoint pass + reverse pass)", "bound": "alu",
                         "achieved": fl / (ms / 1e3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                         "frac": fl / (ms / 1e3) / 1e12 / peak,
                         "peak_source": "148 SMs x 128 fp32 lanes x 2 x max SM clock",
                         "algorithmic_flops_per_launch": fl,
                         "hbm_view": {"algorithmic_bytes": backward_bytes(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv),
                                      "achieved_gbs": backward_bytes(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv)
                                      / (ms / 1e3) / 1e9}}}


def cpu_baseline_table(budget_s=3.0):
    """The fp64 oracle on each workload's recipe, on 1 thread and on all host
    cores: the first two workloads in full, the training shape (forward and
    backward) and the decode workload on samples sized to about `budget_s` each.  Prefill in tokens/s of
    the full workload's head count (token-heads/s / H), decode in GB/s of the
    decode step's algorithmic traffic."""
    import numpy as np

    import oracle
    from gated_delta_rule_100_b200 import inputs

    cores = os.cpu_count() or 1
    rows = []

    def f64(t):
        return t.to("cpu", dtype=__import__("torch").float64).numpy()

    for name in ("oracle_scale_B1_H1_T256_d64", "prefill_B1_H4_T2048_d128", "training_B8_H32_T4096_d128"):
        cfg = inputs.CONFIGS[name]
        for threads in (1, cores):
            full = name != "training_B8_H32_T4096_d128"
            heads = cfg.H if full else min(cfg.H, max(1, threads))
            T = cfg.T
            d = inputs.make_prefill(1 if not full else cfg.B, T, heads, cfg.dk, cfg.dv, decay=cfg.decay,
                                    h0_std=cfg.h0_std, seed=cfg.seed)
            t0 = time.perf_counter()
            oracle.kda_fwd(*(f64(d[k]) for k in ("q", "k", "v", "g", "beta")), cfg.scale,
                           None if d["h0"] is None else f64(d["h0"]), threads=threads)
            dt = time.perf_counter() - t0
            th = d["q"].shape[0] * T * heads
            rows.append({"workload": name, "threads": threads, "seconds": dt,
                         "sample": "full" if full else f"{heads} heads x {T} tokens (batch 1)",
                         "tokens_per_s": th / dt / cfg.H})
    # the backward on the training shape's recipe: the oracle keeps every state of a
    # (b, h), so a sample of 512 tokens per head, one head per thread
    cfg = inputs.CONFIGS["training_B8_H32_T4096_d128"]
    for threads in (1, cores):
        heads, T = min(cfg.H, max(1, threads)), 512
        d = inputs.make_prefill(1, T, heads, cfg.dk, cfg.dv, decay=cfg.decay, h0_std=cfg.h0_std, seed=cfg.seed)
        gen = __import__("torch").Generator().manual_seed(cfg.seed + 100)
        dout = __import__("torch").randn((1, T, heads, cfg.dv), generator=gen)
        t0 = time.perf_counter()
        oracle.kda_bwd(*(f64(d[k]) for k in ("q", "k", "v", "g", "beta")), cfg.scale,
                       None if d["h0"] is None else f64(d["h0"]), f64(dout), None, threads=threads)
        dt = time.perf_counter() - t0
        rows.append({"workload": cfg.name + " backward", "threads": threads, "seconds": dt,
                     "sample": f"{heads} heads x {T} tokens (batch 1)", "tokens_per_s": T * heads / dt / cfg.H})
    dcfg = inputs.DECODE_CONFIG
    for threads in (1, cores):
        nbh = min(dcfg.B, 8 * max(1, threads))  # sequences of the sample (all heads of each)
        d = inputs.make_decode(nbh, dcfg.H, dcfg.dk, dcfg.dv, decay=dcfg.decay, state_std=dcfg.state_std,
                               steps=8, seed=dcfg.seed)
        S = f64(d["state"])
        t0 = time.perf_counter()
        for s_ in range(8):
            _, S = oracle.kda_decode_step(*(f64(d[k][s_]) for k in ("q", "k", "v", "g", "beta")), dcfg.scale, S,
                                          threads=threads)
        dt = time.perf_counter() - t0
        gbs = decode_bytes(nbh, dcfg.H, dcfg.dk, dcfg.dv) * 8 / dt / 1e9
        rows.append({"workload": dcfg.name, "threads": threads, "seconds": dt,
                     "sample": f"{nbh} of {dcfg.B} sequences x {dcfg.H} heads x 8 steps", "state_gbs": gbs})
    del np
    return {"kind": "oracle", "cores": cores, "rows": rows,
            "note": "fp64 oracle; OpenMP over (b, h), so a workload with fewer (b, h) than threads uses fewer"}


# -------------------------------------------------------------------- arms ----
def run_reference(args):
    """The fp64 oracle on the host cores (rank 0 only)."""
    import torch
    from gated_delta_rule_100_b200 import inputs

    world, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    cfg = inputs.CONFIGS[WORKLOAD]
    cores = os.cpu_count() or 1
    heads = min(cfg.H, cores)
    tokens = 2048
    d = inputs.make_prefill(cfg.B, tokens, heads, cfg.dk, cfg.dv, decay=cfg.decay, seed=cfg.seed)
    times = []
    for i in range(args.warmup + args.steps):
        dt, n = oracle_rate(d, cfg.scale, heads, tokens, heads)
        if i >= args.warmup:
            times.append(dt)
    step = statistics.mean(times)
    value = heads * tokens / step / cfg.H
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": cfg.B, "H": cfg.H, "T": cfg.T, "dk": cfg.dk, "dv": cfg.dv},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": heads, "kind": "oracle",
                         "sample": f"each step: fp64 oracle on {heads} heads x {tokens} tokens "
                                   f"(synthetic, workload recipe); tokens/s = token-heads/s / {cfg.H}"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch

    from gated_delta_rule_100_b200 import inputs, kda

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kda.load()
    cfg = inputs.CONFIGS[args.workload]
    P, peak_src = peaks()
    stream = torch.cuda.current_stream()

    # ---------------- prefill (the step) ----------------
    d = inputs.make_config(cfg, device=dev) if rank == 0 else inputs.make_prefill(
        cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, decay=cfg.decay, h0_std=cfg.h0_std, seed=cfg.seed + 1000 * rank,
        device=dev)
    out = torch.empty((cfg.B, cfg.T, cfg.H, cfg.dv), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((cfg.B, cfg.H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)

    def step():
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], cfg.scale, d["h0"], out=out, hT=hT,
                      stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if kda.stream_status(stream) != kda.KDA_OK:
        raise RuntimeError("device-side error during warm-up")

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(args.steps):
            step()
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    if kda.stream_status(stream) != kda.KDA_OK:
        raise RuntimeError("device-side error in the timed region")
    launch_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    # Per-kernel split and launch count: one more step, outside the timed region,
    # with every launch's busy interval stamped by its own CTAs (%globaltimer).
    kda.kernel_times()
    kda.kernel_timing(True)
    step()
    torch.cuda.synchronize()
    kda.kernel_timing(False)
    ktimes = kda.kernel_times()
    total_ms = ev[0].elapsed_time(ev[-1])
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    tokens_per_step = cfg.B * cfg.T
    value = weak_value(tokens_per_step, world, args.steps, total_ms)

    nbytes = prefill_bytes(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.h0_std > 0, True)
    nflops = prefill_flops(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv)
    avg_launch_s = statistics.mean(launch_ms) / 1e3
    achieved = nbytes / avg_launch_s / 1e9
    kernels = {k: {"ms_per_step": t, "launches_per_step": n, "busy_fraction_of_step": t / ms_per_step}
               for k, (t, n) in ktimes.items() if n > 0}
    kernels["note"] = ("per kind: the launches' busy intervals (first CTA start to last CTA end, stamped by the "
                       "kernels) summed over one extra step; prep and chain launches overlap on two streams")
    gpu_launches = sum(n for _, n in ktimes.values()) * args.steps
    th_step = cfg.B * cfg.T * cfg.H
    bpth = [measured_traffic(k, "bytes_per_token_head") for k in ("prep_kernel", "chain_kernel")]
    traffic = traffic_note = None
    if all(b is not None for b, _ in bpth):
        traffic = sum(b for b, _ in bpth) * th_step
        traffic_note = (f"DRAM bytes of prep_kernel + chain_kernel per token-head, captured by ncu on "
                        f"{bpth[0][1]} (the same segmented two-stream code path), times this workload's "
                        f"token-heads: a scaled estimate, not a capture of this workload")
    roof = {"kernel": "kda_chunk_fwd (prep_kernel + chain_kernel)", "bound": "hbm", "achieved": achieved,
            "peak": P["hbm_gbs"], "unit": "GB/s", "frac": achieved / P["hbm_gbs"], "peak_source": peak_src,
            "traffic": traffic, "traffic_note": traffic_note,
            "algorithmic_bytes_per_launch": nbytes, "kernels": kernels,
            "tensor_view": {"achieved_tflops": nflops / avg_launch_s / 1e12,
                            "peak_tflops": P["bf16_tflops_sustained"],
                            "frac": nflops / avg_launch_s / 1e12 / P["bf16_tflops_sustained"]}}

    # ---------------- scalar-gate form (after the timed steps; never fails the line) ----------------
    gdn = None
    if not args.no_gdn:
        try:
            gdn = measure_scalar_gate(d, cfg, out, hT, stream, args.steps, args.warmup, P)
        except Exception as exc:  # noqa: BLE001 - an extra item must not cost the measurement above
            gdn = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    # ---------------- training shape (after the timed steps; never fails the line) ----------------
    training = None
    if not args.no_training:
        try:
            training = measure_training(P, peak_src, stream, args.steps, args.warmup, dev)
        except Exception as exc:  # noqa: BLE001 - an extra item must not cost the measurement above
            training = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    raw = None
    if not args.no_raw:
        try:
            raw = measure_raw(d, cfg, out, hT, stream, args.steps, args.warmup, P)
        except Exception as exc:  # noqa: BLE001 - an extra item must not cost the measurement above
            raw = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    varlen = None
    if not args.no_varlen:
        try:
            varlen = measure_varlen(stream, args.steps, args.warmup, P, dev)
        except Exception as exc:  # noqa: BLE001
            varlen = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    two_level = None
    if not args.no_two_level:
        try:
            two_level = measure_two_level(stream, args.steps, args.warmup, P, dev)
        except Exception as exc:  # noqa: BLE001
            two_level = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    backward = None
    if not args.no_backward:
        try:
            backward = measure_backward(P, stream, args.steps, dev)
        except Exception as exc:  # noqa: BLE001
            backward = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    # ---------------- decode ----------------
    dec = None
    if not args.no_decode:
        dcfg = inputs.DECODE_CONFIG
        dd = inputs.make_decode_config(dcfg, device=dev)
        state = dd["state"]
        dout = torch.empty((dcfg.B, dcfg.H, dcfg.dv), dtype=torch.bfloat16, device=dev)
        for s in range(3):
            kda.decode_step(dd["q"][s], dd["k"][s], dd["v"][s], dd["g"][s], dd["beta"][s], dcfg.scale, state,
                            out=dout, stream=stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        e0.record(stream)
        for s in range(dcfg.steps):
            kda.decode_step(dd["q"][s], dd["k"][s], dd["v"][s], dd["g"][s], dd["beta"][s], dcfg.scale, state,
                            out=dout, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        dms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        db = decode_bytes(dcfg.B, dcfg.H, dcfg.dk, dcfg.dv)
        gbs = db * dcfg.steps / (dms / 1e3) / 1e9
        dec = {"metric": "decode-step state GB/s", "value": gbs * world, "unit": "GB/s",
               "per_gpu_gbs": gbs, "us_per_step": dms * 1e3 / dcfg.steps, "steps": dcfg.steps,
               "config": {"workload": dcfg.name, "B": dcfg.B, "H": dcfg.H, "dk": dcfg.dk, "dv": dcfg.dv},
               "gpu_launches": dcfg.steps,
               "roofline": {"kernel": "decode_step_kernel", "bound": "hbm", "achieved": gbs,
                            "peak": P["hbm_gbs"], "unit": "GB/s", "frac": gbs / P["hbm_gbs"],
                            "peak_source": peak_src,
                            "traffic": measured_traffic("decode_step_kernel")[0],
                            "traffic_note": "ncu dram__bytes_read.sum + dram__bytes_write.sum per launch, "
                                            "captured on this workload",
                            "algorithmic_bytes_per_launch": db}}
        # the same steps from raw projections (gate prologue and q/k norms in the kernel),
        # the workload's tensors taken as the raw values; it never fails the line
        try:
            def raw_step(s):
                kda.decode_step_raw(dd["q"][s], dd["k"][s], dd["v"][s], dd["g"][s], dd["beta"][s], dcfg.decay,
                                    dcfg.scale, state, out=dout, stream=stream)

            for s in range(3):
                raw_step(s)
            torch.cuda.synchronize()
            e0.record(stream)
            for s in range(dcfg.steps):
                raw_step(s)
            e1.record(stream)
            torch.cuda.synchronize()
            if kda.stream_status(stream) != kda.KDA_OK:
                raise RuntimeError("device-side error in the raw decode steps")
            rms = e0.elapsed_time(e1)
            rgbs = db * dcfg.steps / (rms / 1e3) / 1e9
            dec["raw_prologue"] = {"entry_point": "kda_decode_step_raw", "us_per_step": rms * 1e3 / dcfg.steps,
                                   "achieved_gbs": rgbs, "frac": rgbs / P["hbm_gbs"], "gate_c": dcfg.decay}
        except Exception as exc:  # noqa: BLE001
            dec["raw_prologue"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        del dd, state

    # ---------------- end to end from pinned host buffers ----------------
    e2e = None
    if not args.no_e2e:
        host = {k: (torch.empty(v.shape, dtype=v.dtype, pin_memory=True).copy_(v) if v is not None else None)
                for k, v in d.items()}
        h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        h_hT = torch.empty(hT.shape, dtype=hT.dtype, pin_memory=True)
        e2e_steps = max(1, min(args.steps, 3))
        nin = nout = 0
        kda.chunk_fwd_host(host["q"], host["k"], host["v"], host["g"], host["beta"], cfg.scale, host["h0"],
                           out=h_out, hT=h_hT, stream=stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        e0.record(stream)
        for _ in range(e2e_steps):
            nin, nout = kda.chunk_fwd_host(host["q"], host["k"], host["v"], host["g"], host["beta"], cfg.scale,
                                           host["h0"], out=h_out, hT=h_hT, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ems = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": tokens_per_step * world * e2e_steps / (ems / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": nin, "d2h_bytes_per_step": nout, "steps": e2e_steps,
               "ms_per_step": ems / e2e_steps}
        del host, h_out, h_hT

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(d, cfg, args.cpu_seconds)
        try:
            cpu["per_workload"] = cpu_baseline_table()
        except Exception as exc:  # noqa: BLE001
            cpu["per_workload"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "B": cfg.B, "H": cfg.H, "T": cfg.T, "dk": cfg.dk,
                       "dv": cfg.dv, "chunk": CHUNK, "seed": cfg.seed,
                       "operands": "bf16 q/k/v, fp32 g/beta/state; tcgen05 bf16, fp16 and tf32 MMA, fp32 accumulate",
                       "l2": "inputs larger than L2 (51.7 GB per step); no flush",
                       "parallelism": f"weak: one workload copy per GPU x{world}"},
            "tflops": nflops / (ms_per_step / 1e3) / 1e12 * world,
            "roofline": roof, "decode": dec, "scalar_gate": gdn, "training": training, "backward": backward,
            "raw_prologue": raw, "varlen": varlen, "two_level": two_level,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "clocks": clk.summary(), "gpu_launches": gpu_launches,
            "launch_ms": {"mean": statistics.mean(launch_ms), "min": min(launch_ms), "max": max(launch_ms)},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-gdn", action="store_true", help="skip the scalar-gate prefill line")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-training", action="store_true", help="skip the training-shape prefill line")
    ap.add_argument("--no-backward", action="store_true", help="skip the training-shape backward line")
    ap.add_argument("--no-raw", action="store_true", help="skip the raw-input (gate prologue) prefill line")
    ap.add_argument("--no-varlen", action="store_true", help="skip the packed-batch prefill line")
    ap.add_argument("--no-two-level", action="store_true", help="skip the few-heads long-sequence line")
    ap.add_argument("--record-traffic", metavar="CSV",
                    help="write profiles/traffic.json from an ncu dram-bytes CSV and exit")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    if args.record_traffic:
        print(json.dumps(record_traffic(args.record_traffic, args.workload), indent=1))
        return 0
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    return run_reference(args) if args.impl == "reference" else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
