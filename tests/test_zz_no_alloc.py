"""kda_chunk_fwd_noalloc -- the prefill over the library's fixed 64 MiB scratch
array (no device allocation) -- against kda_chunk_fwd on the same inputs.

Both run the same two kernels; only the segmentation of the sequence differs
(the fixed array holds fewer chunk records per segment), and the state carried
between segments is the same fp32 values either way, so the outputs must be
bit-identical.  Two calls in a row check that nothing left in the scratch by
one call changes the next.  Called through the C ABI (ctypes); this file is
collected last so it also runs after every other GPU test."""
import ctypes

import pytest
import torch

from gated_delta_rule_100_b200 import inputs, kda

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, d, scale, out, hT):
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.kda_chunk_fwd_noalloc(_p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["g"]), _p(d["beta"]),
                                     float(scale), _p(d["h0"]), _p(out), _p(hT), B, T, H, dk, dv, stream)


@pytest.mark.parametrize("B,T,H,dk,dv,with_hT", [
    (2, 1000, 64, 128, 128, True),   # 128 (b, h): 5 chunks per segment -> 4 segments, ragged tail
    (2, 1000, 64, 128, 128, False),  # state carried in the scratch: 4 chunks per segment
    (1, 300, 3, 64, 128, True),      # one segment
    (3, 130, 5, 128, 64, False),
])
def test_noalloc_matches_chunk_fwd_twice(B, T, H, dk, dv, with_hT):
    lib = kda.load()
    dev = torch.device("cuda", 0)
    d = inputs.make_prefill(B, T, H, dk, dv, decay=0.05, h0_std=0.02, seed=11, device=dev)
    scale = dk ** -0.5
    ref_out, ref_hT = kda.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], scale, d["h0"])
    assert kda.stream_status() == kda.KDA_OK
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        hT = torch.full_like(ref_hT, float("nan")) if with_hT else None
        rc = _noalloc(lib, d, scale, out, hT)
        assert rc == kda.KDA_OK, kda.status_string(rc)
        assert kda.stream_status() == kda.KDA_OK
        assert torch.equal(out, ref_out)
        if with_hT:
            assert torch.equal(hT, ref_hT)


def test_noalloc_allocates_nothing():
    """With the prefill workspace released, a warmed-up kda_chunk_fwd_noalloc call
    must leave the device's free memory unchanged: no cudaMalloc of a workspace
    (which would be at least the 64 MiB of records this problem needs), nothing
    else either."""
    lib = kda.load()
    dev = torch.device("cuda", 0)
    d = inputs.make_prefill(2, 1000, 64, 128, 128, decay=0.05, h0_std=0.02, seed=12, device=dev)
    out = torch.empty((2, 1000, 64, 128), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((2, 64, 128, 128), dtype=torch.float32, device=dev)
    assert _noalloc(lib, d, 128 ** -0.5, out, hT) == kda.KDA_OK  # first call: symbol lookup, lazy loading
    torch.cuda.synchronize()
    kda.release_workspace()
    assert kda.workspace_bytes(2, 1000, 64, 128, 128) >= 64 << 20
    free0, _ = torch.cuda.mem_get_info(dev)
    for _ in range(2):
        assert _noalloc(lib, d, 128 ** -0.5, out, hT) == kda.KDA_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(dev)
    assert kda.stream_status() == kda.KDA_OK
    assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"


def test_noalloc_zero_length_and_limit():
    lib = kda.load()
    dev = torch.device("cuda", 0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    h0 = torch.randn((1, 2, 64, 64), device=dev)
    hT = torch.full_like(h0, float("nan"))
    # T == 0: no token to scan, hT = h0; the data pointers may be NULL
    rc = lib.kda_chunk_fwd_noalloc(None, None, None, None, None, 0.125, _p(h0), None, _p(hT), 1, 0, 2, 64, 64,
                                   stream)
    assert rc == kda.KDA_OK
    torch.cuda.synchronize()
    assert torch.equal(hT, h0)
    # one chunk record of each of 904 (b, h) exceeds the 64 MiB array: rejected, nothing enqueued
    big = inputs.make_prefill(1, 64, 904, 128, 128, decay=0.05, h0_std=0.0, seed=13, device=dev)
    out = torch.empty((1, 64, 904, 128), dtype=torch.bfloat16, device=dev)
    hT2 = torch.empty((1, 904, 128, 128), dtype=torch.float32, device=dev)
    assert _noalloc(lib, big, 0.1, out, hT2) == kda.KDA_ERR_SCRATCH_LIMIT
