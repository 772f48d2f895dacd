"""kda_chunk_fwd_host, the prefill on host buffers (pieces of the token axis streamed
up, through kda_chunk_fwd and back), through the C ABI: against kda_chunk_fwd on
device copies of the same inputs, and against the fp64 oracle."""
import numpy as np
import pytest
import torch

from gated_delta_rule_100_b200 import inputs, kda
from kda_testlib import assert_close, oracle_prefill

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _reset_hooks():
    kda.set_host_piece(0)
    yield
    kda.set_host_piece(0)


def host_copy(d, pinned=True):
    return {k: (None if v is None else torch.empty(v.shape, dtype=v.dtype, pin_memory=pinned).copy_(v.cpu()))
            for k, v in d.items()}


def run_host(h, scale, want_hT=True, pinned=True):
    B, T, H, _ = h["q"].shape
    dv, dk = h["v"].shape[-1], h["q"].shape[-1]
    out = torch.empty((B, T, H, dv), dtype=torch.bfloat16, pin_memory=pinned)
    hT = torch.empty((B, H, dk, dv), dtype=torch.float32, pin_memory=pinned) if want_hT else None
    nin, nout = kda.chunk_fwd_host(h["q"], h["k"], h["v"], h["g"], h["beta"], scale, h["h0"], out=out, hT=hT)
    torch.cuda.synchronize()
    assert kda.stream_status() == kda.KDA_OK
    return out, hT, nin, nout


def run_device(d, scale):
    out, hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale, d["h0"])
    torch.cuda.synchronize()
    return out.cpu(), hT.cpu()


@pytest.mark.parametrize("piece", [64, 192, 448])
def test_host_pieces_match_device_call(piece):
    """Pieces of whole chunks: every chunk is the device call's chunk and the state
    crosses piece boundaries in fp32, so out and hT are bit-identical."""
    d = inputs.make_prefill(2, 1000, 3, 128, 128, decay=0.05, h0_std=0.02, seed=700, device=DEV)
    kda.set_host_piece(piece)
    out, hT, nin, nout = run_host(host_copy(d), 0.1)
    ref_out, ref_hT = run_device(d, 0.1)
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(hT, ref_hT)
    assert nin == sum(t.numel() * t.element_size() for t in d.values() if t is not None)
    assert nout == out.numel() * 2 + hT.numel() * 4


@pytest.mark.parametrize("piece", [1, 100, 333])
def test_host_ragged_pieces_match_oracle(piece):
    """Piece boundaries inside chunks (a test-only size): the result is the same
    recurrence, checked against the oracle at the parity bar."""
    d = inputs.make_prefill(1, 700, 2, 128, 128, decay=0.05, h0_std=0.02, seed=701 + piece, device=DEV)
    kda.set_host_piece(piece)
    out, hT, _, _ = run_host(host_copy(d), 0.1)
    ref_out, ref_hT = oracle_prefill(d, 0.1)
    assert_close(out.float().numpy(), ref_out, f"host piece {piece} out")
    assert_close(hT.numpy(), ref_hT, f"host piece {piece} hT")


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_host_head_dims(dk, dv):
    d = inputs.make_prefill(1, 500, 4, dk, dv, decay=0.05, h0_std=0.02, seed=710 + dk + dv, device=DEV)
    kda.set_host_piece(128)
    out, hT, _, _ = run_host(host_copy(d), dk ** -0.5)
    ref_out, ref_hT = run_device(d, dk ** -0.5)
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(hT, ref_hT)


def test_host_without_h0_or_hT_and_pageable():
    """No initial state, no final state requested, pageable host memory."""
    d = inputs.make_prefill(1, 300, 2, 128, 128, decay=0.05, seed=720, device=DEV)
    assert d["h0"] is None
    kda.set_host_piece(128)
    out, hT, _, _ = run_host(host_copy(d, pinned=False), 0.1, want_hT=False, pinned=False)
    assert hT is None
    ref_out, _ = run_device(d, 0.1)
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))


def test_host_automatic_pieces_long():
    """The automatic piece size (about 256 MB of inputs: 6,528 tokens here) on a
    sequence of several pieces, sampled against the oracle on two heads."""
    d = inputs.make_prefill(1, 20000, 32, 128, 128, decay=0.01, seed=730, device=DEV)
    out, hT, _, _ = run_host(host_copy(d), 128 ** -0.5)
    ref_out, ref_hT = run_device(d, 128 ** -0.5)
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert torch.equal(hT, ref_hT)
    o_ref, s_ref = oracle_prefill(d, 128 ** -0.5, heads=slice(0, 2))
    assert_close(out[:, :, 0:2].float().numpy(), o_ref, "host automatic pieces out (heads 0-1)")
    assert_close(hT[:, 0:2].numpy(), s_ref, "host automatic pieces hT (heads 0-1)")


def test_host_empty_sequence():
    """T == 0: hT = h0 (or zero), written on the host once the stream is idle."""
    B, H = 2, 3
    h0 = torch.randn((B, H, 128, 128), dtype=torch.float32).pin_memory()
    q = torch.empty((B, 0, H, 128), dtype=torch.bfloat16)
    g = torch.empty((B, 0, H, 128), dtype=torch.float32)
    beta = torch.empty((B, 0, H), dtype=torch.float32)
    out = torch.empty((B, 0, H, 128), dtype=torch.bfloat16)
    hT = torch.full((B, H, 128, 128), 7.0)
    kda.chunk_fwd_host(q, q, q, g, beta, 0.1, h0, out=out, hT=hT)
    assert torch.equal(hT, h0)
    kda.chunk_fwd_host(q, q, q, g, beta, 0.1, None, out=out, hT=hT)
    assert torch.count_nonzero(hT) == 0


def test_host_calls_back_to_back_reuse_staging():
    """Two calls on different inputs, enqueued without a synchronisation between
    them, share the library's staging: each gets its own results."""
    kda.set_host_piece(128)
    d1 = inputs.make_prefill(1, 600, 2, 128, 128, decay=0.05, h0_std=0.02, seed=740, device=DEV)
    d2 = inputs.make_prefill(1, 600, 2, 128, 128, decay=0.05, h0_std=0.02, seed=741, device=DEV)
    h1, h2 = host_copy(d1), host_copy(d2)
    outs = [torch.empty((1, 600, 2, 128), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hTs = [torch.empty((1, 2, 128, 128), dtype=torch.float32).pin_memory() for _ in range(2)]
    for h, o, s in zip((h1, h2), outs, hTs):
        kda.chunk_fwd_host(h["q"], h["k"], h["v"], h["g"], h["beta"], 0.1, h["h0"], out=o, hT=s)
    torch.cuda.synchronize()
    for d, o, s in zip((d1, d2), outs, hTs):
        ref_out, ref_hT = run_device(d, 0.1)
        assert torch.equal(o.view(torch.int16), ref_out.view(torch.int16))
        assert torch.equal(s, ref_hT)
    assert not np.array_equal(outs[0].float().numpy(), outs[1].float().numpy())
