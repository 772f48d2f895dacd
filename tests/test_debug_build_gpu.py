"""libkda_debug.so, the build with device-side index checks (KDA_DEBUG): every
record index and offset, shared-memory tile and tensor-operand view, token row
and state slice whose bounds rest on layout constants and launch geometry is
checked before use; a failed check is reported as KDA_ERR_BOUNDS (the access
is skipped, nothing traps).  Run through the same binding on the small
workload, short and ragged lengths, every path of the prefill (exact, block
references, two-level, segmented, packed with windows, no-allocation, raw inputs, scalar
gate) and the backward: no check may fail, and the results must still match
the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_100_b200 import inputs, kda
from kda_testlib import assert_close, f64, oracle_prefill

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _reset():
    kda.set_parts(0)
    kda.set_record_cap(0)
    kda.force_exact(False)
    kda.block_refs(False)


@pytest.fixture(autouse=True)
def debug_library():
    kda.use_debug_library(True)
    _reset()
    yield
    _reset()
    kda.use_debug_library(False)


def run_and_check(d, scale, what, **kw):
    out, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale, d["h0"], **kw)
    assert kda.stream_status() == kda.KDA_OK, f"{what}: an index check failed"
    o_ref, s_ref = oracle_prefill(d, scale)
    assert_close(f64(out), o_ref, f"debug build {what} out")
    if hT is not None:
        assert_close(f64(hT), s_ref, f"debug build {what} hT")


def test_small_workload():
    cfg = inputs.CONFIGS["oracle_scale_B1_H1_T256_d64"]
    run_and_check(inputs.make_config(cfg, device=DEV), cfg.scale, cfg.name)


@pytest.mark.parametrize("T", [1, 15, 63, 64, 65])
@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (128, 128)])
def test_short_lengths(T, dk, dv):
    d = inputs.make_prefill(2, T, 2, dk, dv, decay=0.05, h0_std=0.02, seed=3000 + T, device=DEV)
    run_and_check(d, dk ** -0.5, f"T={T} {dk}x{dv}")


def test_exact_two_level_and_segmented_paths():
    d = inputs.make_prefill(1, 1500, 2, 128, 128, decay=0.05, h0_std=0.02, seed=3100, device=DEV)
    kda.force_exact(True)
    run_and_check(d, 0.1, "exact path")
    kda.force_exact(False)
    kda.block_refs(True)
    run_and_check(d, 0.1, "block references")
    kda.block_refs(False)
    kda.set_parts(3)
    run_and_check(d, 0.1, "two-level pass")
    kda.set_record_cap(2 * 2 * 8 * 74240)
    run_and_check(d, 0.1, "segmented two-level pass")
    kda.set_parts(1)
    run_and_check(d, 0.1, "segmented plain pass", final_state=False)


def test_packed_batch_in_windows():
    lengths = [65, 0, 130, 1, 64]
    T = sum(lengths)
    d = inputs.make_prefill(1, T, 2, 128, 128, decay=0.05, h0_std=0.0, seed=3200, device=DEV)
    d = {k: (v[0] if v is not None else None) for k, v in d.items()}
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device=DEV)
    kda.set_record_cap(2 * 2 * 74240)
    out, hT = kda.chunk_fwd_varlen(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.2, cu)
    assert kda.stream_status() == kda.KDA_OK
    cuh = cu.cpu().tolist()
    for n in range(len(lengths)):
        a, b = cuh[n], cuh[n + 1]
        o, s = oracle.kda_fwd(*(f64(d[k][a:b])[None] for k in ("q", "k", "v", "g", "beta")), 0.2, None)
        if b > a:
            assert_close(f64(out[a:b]), o[0], f"debug varlen seq {n} out")
        assert_close(f64(hT[n]), s[0], f"debug varlen seq {n} hT")


def test_noalloc_raw_and_scalar_gate():
    d = inputs.make_prefill(2, 200, 3, 128, 128, decay=0.05, h0_std=0.02, seed=3300, device=DEV)
    out = torch.empty((2, 200, 3, 128), dtype=torch.bfloat16, device=DEV)
    kda.chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.1, d["h0"], out=out)
    assert kda.stream_status() == kda.KDA_OK
    assert_close(f64(out), oracle_prefill(d, 0.1)[0], "debug noalloc out")
    gs = d["g"][..., 0].contiguous()
    kda.gdn_chunk_fwd(d["q"], d["k"], d["v"], gs, d["beta"], 0.1, d["h0"])
    kda.chunk_fwd_raw(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.5, 0.1, d["h0"])
    assert kda.stream_status() == kda.KDA_OK


@pytest.mark.parametrize("T", [1, 65, 200])
@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (128, 128)])
def test_backward(T, dk, dv):
    """The backward through the debug library: its checks on the level-1 and level-2
    checkpoint regions, the per-token p buffer and the asynchronous checkpoint
    copies never fail, and the gradients match the oracle."""
    d = inputs.make_prefill(2, T, 2, dk, dv, decay=0.05, h0_std=0.02, seed=3300 + T, device=DEV)
    gen = torch.Generator(device=DEV).manual_seed(3400 + T)
    dout = torch.randn((2, T, 2, dv), generator=gen, device=DEV).to(torch.bfloat16)
    dhT = 0.1 * torch.randn((2, 2, dk, dv), generator=gen, device=DEV)
    r = kda.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dk ** -0.5, d["h0"], dout, dhT)
    torch.cuda.synchronize()
    assert kda.stream_status() == kda.KDA_OK, f"backward T={T} {dk}x{dv}: an index check failed"
    ref = oracle.kda_bwd(f64(d["q"]), f64(d["k"]), f64(d["v"]), f64(d["g"]), f64(d["beta"]), dk ** -0.5,
                         f64(d["h0"]), f64(dout), f64(dhT))
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        # the bf16 gradients: one bf16 spacing of the largest reference value, as the backward's tests
        bar = max(2e-2, 2.0 ** -7 * float(np.abs(ref[n]).max())) if n in ("dq", "dk", "dv") else 2e-2
        assert_close(f64(r[n]), ref[n], f"debug backward T={T} {dk}x{dv} {n}", mabs=bar)
