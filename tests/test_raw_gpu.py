"""kda_chunk_fwd_raw and kda_decode_step_raw, the entry points with the gate
prologue fused (raw projections in), through the C ABI against the fp64 oracle.
The prologue's outputs are computed here from the same raw inputs in fp64:
g = -c softplus(g_raw), beta = sigmoid(beta_raw), q and k divided by their L2
norm over dk (floored at 1e-12)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_100_b200 import kda
from kda_testlib import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def prologue64(q, k, g_raw, beta_raw, c):
    """The prologue in fp64 from the raw tensors (numpy float64 in, out)."""
    def unit(x):
        return x / np.maximum(np.linalg.norm(x, axis=-1, keepdims=True), 1e-12)
    g = -c * np.logaddexp(0.0, g_raw)       # softplus
    beta = 1.0 / (1.0 + np.exp(-beta_raw))  # sigmoid
    return unit(q), unit(k), g, beta


def raw_inputs(B, T, H, dk, dv, seed, qk_scale=3.0):
    gen = torch.Generator(device=DEV).manual_seed(seed)

    def rn(*shape):
        return torch.randn(shape, generator=gen, device=DEV)
    return dict(q=(qk_scale * rn(B, T, H, dk)).to(torch.bfloat16), k=(qk_scale * rn(B, T, H, dk)).to(torch.bfloat16),
                v=rn(B, T, H, dv).to(torch.bfloat16), g_raw=rn(B, T, H, dk), beta_raw=rn(B, T, H),
                h0=0.02 * rn(B, H, dk, dv))


@pytest.mark.parametrize("c", [0.05, 1.0, 20.0])
@pytest.mark.parametrize("T", [200, 1000])
def test_prefill_raw(T, c):
    """c = 20 makes the decay steep enough for the exact path, with the prologue."""
    d = raw_inputs(1, T, 2, 128, 128, seed=1000 + T)
    scale = 128 ** -0.5
    out, hT = kda.chunk_fwd_raw(d["q"], d["k"], d["v"], d["g_raw"], d["beta_raw"], c, scale, d["h0"])
    torch.cuda.synchronize()
    assert kda.stream_status() == kda.KDA_OK
    q, k, g, beta = prologue64(f64(d["q"]), f64(d["k"]), f64(d["g_raw"]), f64(d["beta_raw"]), c)
    o_ref, s_ref = oracle.kda_fwd(q, k, f64(d["v"]), g, beta, scale, f64(d["h0"]))
    assert_close(f64(out), o_ref, f"raw prefill c={c} T={T} out")
    assert_close(f64(hT), s_ref, f"raw prefill c={c} T={T} hT")


def test_prefill_raw_matches_unfused():
    """The fused prologue gives what the unfused entry point gives on the prologue's
    values computed on the device (within the parity bar: the rounding points differ)."""
    d = raw_inputs(2, 300, 2, 64, 64, seed=1100)
    c, scale = 0.3, 0.125
    out, hT = kda.chunk_fwd_raw(d["q"], d["k"], d["v"], d["g_raw"], d["beta_raw"], c, scale, d["h0"])
    qn = (d["q"].float() / d["q"].float().norm(dim=-1, keepdim=True).clamp_min(1e-12)).to(torch.bfloat16)
    kn = (d["k"].float() / d["k"].float().norm(dim=-1, keepdim=True).clamp_min(1e-12)).to(torch.bfloat16)
    g = -c * torch.nn.functional.softplus(d["g_raw"])
    out2, hT2 = kda.chunk_fwd(qn, kn, d["v"], g, torch.sigmoid(d["beta_raw"]), scale, d["h0"])
    torch.cuda.synchronize()
    assert_close(f64(out), f64(out2), "raw vs unfused out")
    assert_close(f64(hT), f64(hT2), "raw vs unfused hT")


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
def test_decode_raw(dk, dv):
    steps, c, scale = 6, 0.5, dk ** -0.5
    gen = torch.Generator(device=DEV).manual_seed(1200 + dk)
    B, H = 3, 2
    state = 0.02 * torch.randn((B, H, dk, dv), generator=gen, device=DEV)
    S = f64(state)
    outs, refs = [], []
    for _ in range(steps):
        q = (3 * torch.randn((B, H, dk), generator=gen, device=DEV)).to(torch.bfloat16)
        k = (3 * torch.randn((B, H, dk), generator=gen, device=DEV)).to(torch.bfloat16)
        v = torch.randn((B, H, dv), generator=gen, device=DEV).to(torch.bfloat16)
        gr = torch.randn((B, H, dk), generator=gen, device=DEV)
        br = torch.randn((B, H), generator=gen, device=DEV)
        outs.append(kda.decode_step_raw(q, k, v, gr, br, c, scale, state))
        qq, kk, g, beta = prologue64(f64(q), f64(k), f64(gr), f64(br), c)
        o, S = oracle.kda_decode_step(qq, kk, f64(v), g, beta, scale, S)
        refs.append(o)
    torch.cuda.synchronize()
    assert_close(f64(torch.stack(outs)), np.stack(refs), f"raw decode {dk}x{dv} outputs")
    assert_close(f64(state), np.asarray(S), f"raw decode {dk}x{dv} state")


def test_raw_rejects_bad_gate_scale():
    d = raw_inputs(1, 64, 1, 64, 64, seed=1300)
    for c in (-1.0, float("nan"), float("inf")):
        with pytest.raises(kda.KdaError):
            kda.chunk_fwd_raw(d["q"], d["k"], d["v"], d["g_raw"], d["beta_raw"], c, 0.1)
