"""kda_chunk_bwd, the backward pass of the prefill, through the C ABI against the
fp64 oracle's reverse-mode gradients (kda_oracle_bwd, pinned by finite
differences) on the same bf16-rounded inputs and cotangents."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_100_b200 import inputs, kda
from kda_testlib import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def cotangents(B, T, H, dv, dk, seed, with_dout=True, with_dhT=True):
    gen = torch.Generator(device=DEV).manual_seed(seed)
    dout = torch.randn((B, T, H, dv), generator=gen, device=DEV).to(torch.bfloat16) if with_dout else None
    dhT = torch.randn((B, H, dk, dv), generator=gen, device=DEV) if with_dhT else None
    return dout, dhT


def oracle_grads(d, scale, dout, dhT, threads=None, bsl=slice(None), hsl=slice(None)):
    def cut(t, has_t=True):
        if t is None:
            return None
        return f64(t[bsl, :, hsl] if has_t else t[bsl, hsl])
    return oracle.kda_bwd(cut(d["q"]), cut(d["k"]), cut(d["v"]), cut(d["g"]), cut(d["beta"]), scale,
                          cut(d["h0"], False), cut(dout), cut(dhT, False), threads=threads)


# dq, dk and dv are returned in bf16, like q, k and v: bf16 values near m are
# spaced up to m 2^-7 apart, so storing one can move it by m 2^-8.  Gradients
# are not O(1) like the forward's outputs (dk sums dv products of the state's
# cotangent), so their max-abs bar is the forward's 2e-2 or one bf16 spacing
# of the largest reference value (m 2^-7), whichever is larger; rel-L2 keeps
# its bar.
BF16_GRADS = ("dq", "dk", "dv")


def check(r, ref, what, bsl=slice(None), hsl=slice(None)):
    for name in ("dq", "dk", "dv", "dg", "dbeta"):
        mabs = max(2e-2, 2.0 ** -7 * float(np.max(np.abs(ref[name])))) if name in BF16_GRADS else 2e-2
        assert_close(f64(r[name][bsl, :, hsl]), ref[name], f"{what} {name}", mabs=mabs)
    if r["dh0"] is not None:
        assert_close(f64(r["dh0"][bsl, hsl]), ref["dh0"], f"{what} dh0")


@pytest.mark.parametrize("T", [1, 7, 8, 9, 100, 333])
def test_backward_lengths(T):
    d = inputs.make_prefill(2, T, 2, 128, 128, decay=0.05, h0_std=0.02, seed=2000 + T, device=DEV)
    dout, dhT = cotangents(2, T, 2, 128, 128, seed=T)
    r = kda.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.1, d["h0"], dout, dhT)
    torch.cuda.synchronize()
    check(r, oracle_grads(d, 0.1, dout, dhT), f"T={T}")


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_backward_head_dims(dk, dv):
    d = inputs.make_prefill(1, 150, 3, dk, dv, decay=0.1, h0_std=0.02, seed=2100 + dk + dv, device=DEV)
    dout, dhT = cotangents(1, 150, 3, dv, dk, seed=5)
    r = kda.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], dk ** -0.5, d["h0"], dout, dhT)
    torch.cuda.synchronize()
    check(r, oracle_grads(d, dk ** -0.5, dout, dhT), f"{dk}x{dv}")


@pytest.mark.parametrize("with_dout,with_dhT", [(True, False), (False, True)])
def test_backward_one_cotangent(with_dout, with_dhT):
    """Only dL/dout, or only dL/dhT (and no h0, no dh0 wanted)."""
    d = inputs.make_prefill(2, 90, 2, 128, 128, decay=0.05, h0_std=0.0, seed=2200, device=DEV)
    dout, dhT = cotangents(2, 90, 2, 128, 128, seed=6, with_dout=with_dout, with_dhT=with_dhT)
    r = kda.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.2, None, dout, dhT, want_dh0=False)
    torch.cuda.synchronize()
    assert r["dh0"] is None
    ref = oracle_grads(d, 0.2, dout, dhT)
    if with_dout:
        check(r, ref, "dout only")
    else:
        assert torch.count_nonzero(r["dq"]) == 0  # the readout gets no gradient
        for name in ("dk", "dv", "dg", "dbeta"):
            mabs = max(2e-2, 2.0 ** -7 * float(np.max(np.abs(ref[name])))) if name in BF16_GRADS else 2e-2
            assert_close(f64(r[name]), ref[name], f"dhT only {name}", mabs=mabs)


def test_backward_zero_length():
    d = inputs.make_prefill(1, 0, 2, 64, 64, decay=0.05, h0_std=0.02, seed=2300, device=DEV)
    _, dhT = cotangents(1, 1, 2, 64, 64, seed=7)
    r = kda.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.2, d["h0"], None, dhT)
    torch.cuda.synchronize()
    assert torch.equal(r["dh0"], dhT)


def test_backward_training_shape_sampled():
    """The training shape (B8 H32 T4096) in one launch; the oracle checks batch 0,
    heads 0-1 (the gradients of different (b, h) are independent)."""
    cfg = inputs.CONFIGS["training_B8_H32_T4096_d128"]
    d = inputs.make_config(cfg, device=DEV)
    dout, _ = cotangents(cfg.B, cfg.T, cfg.H, cfg.dv, cfg.dk, seed=8, with_dhT=False)
    r = kda.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], cfg.scale, d["h0"], dout, None)
    torch.cuda.synchronize()
    assert kda.stream_status() == kda.KDA_OK
    bsl, hsl = slice(0, 1), slice(0, 2)
    ref = oracle_grads(d, cfg.scale, dout, None, threads=2, bsl=bsl, hsl=hsl)
    check(r, ref, "training shape (b 0, h 0-1)", bsl=bsl, hsl=hsl)
