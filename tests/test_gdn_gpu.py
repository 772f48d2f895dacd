"""kda_gdn_chunk_fwd and kda_gdn_decode_step, the scalar-gate form (one log-decay
per token and head shared by every key channel), on the GPU through the C ABI:
against the fp64 oracle with the gate broadcast over the key channels, and bit
for bit against the per-channel entry points given that broadcast gate (the
kernels apply the same per-channel arithmetic to the same values)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_100_b200 import inputs, kda
from kda_testlib import assert_close, f64, oracle_prefill

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def scalar_and_broadcast(g):
    """A scalar gate from channel 0 of a per-channel one, and that gate broadcast back."""
    gs = g[..., 0].contiguous()
    return gs, gs.unsqueeze(-1).expand_as(g).contiguous()


@pytest.mark.parametrize("B,T,H,dk,dv", [(1, 200, 2, 64, 64), (2, 130, 3, 128, 128), (1, 1000, 2, 128, 64)])
def test_gdn_prefill(B, T, H, dk, dv):
    d = inputs.make_prefill(B, T, H, dk, dv, decay=0.1, h0_std=0.02, seed=300 + T, device=DEV)
    gs, gfull = scalar_and_broadcast(d["g"])
    scale = dk ** -0.5
    out, hT = kda.gdn_chunk_fwd(d["q"], d["k"], d["v"], gs, d["beta"], scale, d["h0"])
    out_b, hT_b = kda.chunk_fwd(d["q"], d["k"], d["v"], gfull, d["beta"], scale, d["h0"])
    torch.cuda.synchronize()
    assert kda.stream_status() == kda.KDA_OK
    assert torch.equal(out, out_b) and torch.equal(hT, hT_b), "scalar gate differs from its broadcast"
    o_ref, s_ref = oracle_prefill(dict(d, g=gfull), scale)
    assert_close(f64(out), o_ref, "scalar-gate out")
    assert_close(f64(hT), s_ref, "scalar-gate hT")


def test_gdn_prefill_rejects_wrong_gate_shape():
    d = inputs.make_prefill(1, 64, 2, 64, 64, decay=0.1, seed=1, device=DEV)
    with pytest.raises(ValueError):
        kda.gdn_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.125)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128)])
def test_gdn_decode(dk, dv):
    steps, scale = 5, dk ** -0.5
    d = inputs.make_decode(3, 2, dk, dv, decay=0.05, state_std=0.02, steps=steps, seed=41, device=DEV)
    state, state_b = d["state"].clone(), d["state"].clone()
    S = f64(d["state"])
    for s in range(steps):
        gs, gfull = scalar_and_broadcast(d["g"][s])
        o = kda.gdn_decode_step(d["q"][s], d["k"][s], d["v"][s], gs, d["beta"][s], scale, state)
        o_b = kda.decode_step(d["q"][s], d["k"][s], d["v"][s], gfull, d["beta"][s], scale, state_b)
        torch.cuda.synchronize()
        assert torch.equal(o, o_b) and torch.equal(state, state_b), f"step {s}: scalar gate differs"
        o_ref, S = oracle.kda_decode_step(f64(d["q"][s]), f64(d["k"][s]), f64(d["v"][s]), f64(gfull),
                                          f64(d["beta"][s]), scale, S)
        assert_close(f64(o), o_ref, f"step {s} out")
    assert_close(f64(state), np.asarray(S), "final state")
    assert kda.stream_status() == kda.KDA_OK
