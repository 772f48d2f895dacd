"""kda_decode_step (CUDA, through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_100_b200 import inputs, kda
from kda_testlib import assert_close, f64, oracle_prefill

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def run_steps(d, scale, steps):
    state = d["state"].clone()
    outs = []
    for s in range(steps):
        outs.append(kda.decode_step(d["q"][s], d["k"][s], d["v"][s], d["g"][s], d["beta"][s], scale, state))
    torch.cuda.synchronize()
    assert kda.stream_status() == kda.KDA_OK
    return torch.stack(outs), state


def oracle_steps(d, scale, steps):
    S = f64(d["state"])
    outs = []
    for s in range(steps):
        o, S = oracle.kda_decode_step(f64(d["q"][s]), f64(d["k"][s]), f64(d["v"][s]), f64(d["g"][s]),
                                      f64(d["beta"][s]), scale, S)
        outs.append(o)
    return np.stack(outs), S


def test_decode_config_full():
    """B=256, H=32, d=128, 64 steps in place: all outputs and the final state."""
    cfg = inputs.DECODE_CONFIG
    d = inputs.make_decode_config(cfg, device=DEV)
    outs, state = run_steps(d, cfg.scale, cfg.steps)
    o_ref, s_ref = oracle_steps(d, cfg.scale, cfg.steps)
    assert_close(f64(outs), o_ref, "decode outputs")
    assert_close(f64(state), s_ref, "decode state")


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_decode_head_dims(dk, dv):
    d = inputs.make_decode(5, 3, dk, dv, decay=0.1, state_std=0.02, steps=7, seed=3, device=DEV)
    outs, state = run_steps(d, dk ** -0.5, 7)
    o_ref, s_ref = oracle_steps(d, dk ** -0.5, 7)
    assert_close(f64(outs), o_ref, f"decode {dk}x{dv} outputs")
    assert_close(f64(state), s_ref, f"decode {dk}x{dv} state")


def test_prefill_then_decode_matches_longer_prefill():
    """Decode continues a prefill: chunk_fwd over T tokens, then one decode step
    with the next token, equals chunk_fwd over T + 1 tokens."""
    T = 130
    d = inputs.make_prefill(2, T + 1, 3, 128, 128, decay=0.05, h0_std=0.02, seed=21, device=DEV)
    full_o, full_s = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.2, d["h0"])
    head = {k: (v[:, :T].contiguous() if k != "h0" else v) for k, v in d.items()}
    _, state = kda.chunk_fwd(head["q"], head["k"], head["v"], head["g"], head["beta"], 0.2, head["h0"])
    o = kda.decode_step(d["q"][:, T].contiguous(), d["k"][:, T].contiguous(), d["v"][:, T].contiguous(),
                        d["g"][:, T].contiguous(), d["beta"][:, T].contiguous(), 0.2, state)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_prefill(d, 0.2)
    assert_close(f64(o), o_ref[:, T], "decode after prefill out")
    assert_close(f64(state), s_ref, "decode after prefill state")
    assert_close(f64(full_s), s_ref, "longer prefill state")
