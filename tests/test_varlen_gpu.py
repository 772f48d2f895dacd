"""kda_chunk_fwd_varlen, the packed-batch prefill (sequences of different lengths
back to back, cu_seqlens on the device, a state per sequence), through the C ABI
against the fp64 oracle run on each sequence alone."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_100_b200 import inputs, kda
from kda_testlib import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(autouse=True)
def _reset_hooks():
    kda.set_record_cap(0)
    yield
    kda.set_record_cap(0)


def packed(lengths, H, dk, dv, seed, h0_std=0.02):
    """Inputs for sequences of `lengths` packed along the token axis, plus cu_seqlens."""
    T = int(sum(lengths))
    d = inputs.make_prefill(1, T, H, dk, dv, decay=0.05, h0_std=0.0, seed=seed, device=DEV)
    d = {k: (v[0] if v is not None else None) for k, v in d.items()}
    gen = torch.Generator(device=DEV).manual_seed(seed + 1)
    d["h0"] = h0_std * torch.randn((len(lengths), H, dk, dv), generator=gen, device=DEV) if h0_std > 0 else None
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device=DEV)
    return d, cu


def oracle_per_sequence(d, cu, scale):
    outs, states = [], []
    cuh = cu.cpu().numpy()
    for n in range(len(cuh) - 1):
        a, b = int(cuh[n]), int(cuh[n + 1])
        h0 = None if d["h0"] is None else f64(d["h0"][n])[None]
        o, s = oracle.kda_fwd(*(f64(d[k][a:b])[None] for k in ("q", "k", "v", "g", "beta")), scale, h0)
        outs.append(o[0])
        states.append(s[0])
    return np.concatenate(outs, axis=0), np.stack(states)


def run(d, cu, scale, **kw):
    out, hT = kda.chunk_fwd_varlen(d["q"], d["k"], d["v"], d["g"], d["beta"], scale, cu, d["h0"], **kw)
    torch.cuda.synchronize()
    assert kda.stream_status() == kda.KDA_OK
    return out, hT


LENGTHS = [1, 63, 64, 65, 1000, 4096]


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128)])
def test_varlen_mixed_lengths(dk, dv):
    lengths = LENGTHS if dk == 128 else [65, 1, 300, 64]
    d, cu = packed(lengths, 3, dk, dv, seed=900 + dk)
    out, hT = run(d, cu, dk ** -0.5)
    o_ref, s_ref = oracle_per_sequence(d, cu, dk ** -0.5)
    assert_close(f64(out), o_ref, f"varlen {lengths} out")
    assert_close(f64(hT), s_ref, f"varlen {lengths} hT")


def test_varlen_empty_sequences_and_null_h0():
    """Empty sequences pass their state through (zero without h0); the others are
    unaffected by them."""
    lengths = [0, 130, 0, 0, 77, 0]
    d, cu = packed(lengths, 2, 128, 128, seed=910, h0_std=0.0)
    out, hT = run(d, cu, 0.2)
    o_ref, s_ref = oracle_per_sequence(d, cu, 0.2)
    assert_close(f64(out), o_ref, "varlen with empty sequences out")
    assert_close(f64(hT), s_ref, "varlen with empty sequences hT")
    assert torch.count_nonzero(hT[[0, 2, 3, 5]]) == 0


def test_varlen_matches_chunk_fwd_per_sequence():
    """Each sequence of the packed batch gives what kda_chunk_fwd gives it alone."""
    lengths = [200, 64, 513]
    d, cu = packed(lengths, 2, 128, 128, seed=920)
    out, hT = run(d, cu, 0.15)
    cuh = cu.cpu().tolist()
    for n in range(len(lengths)):
        a, b = cuh[n], cuh[n + 1]
        o1, s1 = kda.chunk_fwd(*(d[k][a:b][None].contiguous() for k in ("q", "k", "v", "g", "beta")), 0.15,
                               d["h0"][n][None].contiguous())
        torch.cuda.synchronize()
        assert_close(f64(out[a:b]), f64(o1[0]), f"sequence {n} out vs chunk_fwd")
        assert_close(f64(hT[n]), f64(s1[0]), f"sequence {n} hT vs chunk_fwd")


def test_varlen_windows_give_the_same_bits():
    """With the record cap shrunk to 3 chunks of every head, the packed batch runs
    in many windows, sequences carrying their state across them (in hT, and in the
    workspace when hT is not wanted); the results must equal the one-window run bit
    for bit (same kernels, state carried in fp32)."""
    lengths = [70, 1, 200, 0, 129]
    H = 2
    d, cu = packed(lengths, H, 128, 128, seed=930)
    out1, hT1 = run(d, cu, 0.2)
    kda.set_record_cap(3 * H * 74240)
    out2, hT2 = run(d, cu, 0.2)
    out3, _ = run(d, cu, 0.2, final_state=False)
    assert torch.equal(out1, out2) and torch.equal(hT1, hT2)
    assert torch.equal(out1, out3)
    o_ref, s_ref = oracle_per_sequence(d, cu, 0.2)
    assert_close(f64(out2), o_ref, "windowed out")
    assert_close(f64(hT2), s_ref, "windowed hT")


def test_segmented_uniform_path_gives_the_same_bits():
    """The same record cap splits a uniform batch into segments of 2 chunks on two
    streams (the path of long sequences): the results must equal one segment's."""
    d = inputs.make_prefill(2, 700, 2, 128, 128, decay=0.05, h0_std=0.02, seed=940, device=DEV)
    o1, s1 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.2, d["h0"])
    kda.set_record_cap(4 * 4 * 74240)  # two buffers of 2 chunks of the 4 (b, h)
    o2, s2 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.2, d["h0"])
    o3, _ = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.2, d["h0"], final_state=False)
    torch.cuda.synchronize()
    assert kda.stream_status() == kda.KDA_OK
    assert torch.equal(o1, o2) and torch.equal(s1, s2) and torch.equal(o1, o3)


def test_varlen_bad_offsets_are_reported_not_faulting():
    """Offsets that decrease or pass T_total are clamped on the device before use
    and reported as KDA_ERR_INVALID_ARG by kda_stream_status."""
    d, cu = packed([100, 50], 2, 64, 64, seed=950)
    bad = torch.tensor([0, 120, 90], dtype=torch.int32, device=DEV)  # decreases, ends short
    kda.chunk_fwd_varlen(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.2, bad, d["h0"])
    assert kda.stream_status() == kda.KDA_ERR_INVALID_ARG
    bad2 = torch.tensor([0, 100, 1000], dtype=torch.int32, device=DEV)  # past T_total
    kda.chunk_fwd_varlen(d["q"], d["k"], d["v"], d["g"], d["beta"], 0.2, bad2, d["h0"])
    assert kda.stream_status() == kda.KDA_ERR_INVALID_ARG
    run(d, cu, 0.2)  # a good call afterwards is clean
