"""The C ABI loads on a CPU-only host, exports what include/kda.h declares, and
rejects bad arguments before touching a GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_100_b200 import build as kbuild
from gated_delta_rule_100_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load()


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"KDA_API\s+[\w\s\*]*?\b(kda_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    assert "kda_chunk_fwd" in names and "kda_decode_step" in names
    assert set(names) == set(kda.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.kda_abi_version() == 104


def test_status_strings(lib):
    for code, name in enumerate(["KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED",
                                 "KDA_ERR_ALIGNMENT", "KDA_ERR_CUDA", "KDA_ERR_TIMEOUT"]):
        assert kda.status_string(code) == name
    assert kda.status_string(99) == "KDA_ERR_UNKNOWN"


A = ctypes.c_void_p(0x10000)     # stand-in device addresses: only validated, never dereferenced
MIS = ctypes.c_void_p(0x10008)   # 8-byte aligned, not 16
ODD = ctypes.c_void_p(0x10002)   # 2-byte aligned


def chunk(lib, q=A, k=A, v=A, g=A, beta=A, h0=None, out=A, hT=None, B=1, T=64, H=1, dk=64, dv=64):
    return lib.kda_chunk_fwd(q, k, v, g, beta, 1.0, h0, out, hT, B, T, H, dk, dv, None)


def decode(lib, q=A, k=A, v=A, g=A, beta=A, state=A, out=A, B=1, H=1, dk=64, dv=64):
    return lib.kda_decode_step(q, k, v, g, beta, 1.0, state, out, B, H, dk, dv, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(beta=None), kda.KDA_ERR_INVALID_ARG),
    (dict(out=None), kda.KDA_ERR_INVALID_ARG),
    (dict(B=0), kda.KDA_ERR_INVALID_ARG),
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(B=0, T=0), kda.KDA_ERR_INVALID_ARG),
    (dict(T=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(dv=256), kda.KDA_ERR_UNSUPPORTED),
    (dict(k=MIS), kda.KDA_ERR_ALIGNMENT),
    (dict(beta=ODD), kda.KDA_ERR_ALIGNMENT),
    (dict(h0=MIS), kda.KDA_ERR_ALIGNMENT),
    (dict(hT=MIS), kda.KDA_ERR_ALIGNMENT),
])
def test_chunk_fwd_rejects(lib, kw, code):
    assert chunk(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(state=None), kda.KDA_ERR_INVALID_ARG),
    (dict(out=None), kda.KDA_ERR_INVALID_ARG),
    (dict(B=0), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(v=MIS), kda.KDA_ERR_ALIGNMENT),
    (dict(beta=ODD), kda.KDA_ERR_ALIGNMENT),
])
def test_decode_step_rejects(lib, kw, code):
    assert decode(lib, **kw) == code


def host_chunk(lib, q=A, k=A, v=A, g=A, beta=A, h0=None, out=A, hT=None, B=1, T=64, H=1, dk=64, dv=64):
    return lib.kda_chunk_fwd_host(q, k, v, g, beta, 1.0, h0, out, hT, B, T, H, dk, dv, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(g=None), kda.KDA_ERR_INVALID_ARG),
    (dict(out=None), kda.KDA_ERR_INVALID_ARG),
    (dict(B=0), kda.KDA_ERR_INVALID_ARG),
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(T=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(dv=32), kda.KDA_ERR_UNSUPPORTED),
])
def test_chunk_fwd_host_rejects(lib, kw, code):
    # validated before any CUDA call (host pointers need no alignment)
    assert host_chunk(lib, **kw) == code


def test_zero_length_accepts_null_inputs(lib):
    # T == 0 with no h0/hT: nothing to read or write, so nothing is enqueued
    assert chunk(lib, q=None, k=None, v=None, g=None, beta=None, out=None, T=0) == kda.KDA_OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(kda, "_lib", None)
    monkeypatch.setattr(kda, "LIB_PATH", str(tmp_path / "libkda.so"))
    with pytest.raises(RuntimeError, match="missing"):
        kda.load()


def test_workspace_bytes(lib):
    rec = 74240  # bytes of one chunk record of one (b, h)
    tick = 256   # the prep kernel's item and steep-item counters

    def lst(items):  # the list of steep items: one int per item of a segment, 256-byte rounded
        return (4 * items + 255) // 256 * 256

    # one segment: all chunks' records, no state buffer
    assert kda.workspace_bytes(1, 256, 1, 128, 128) == tick + lst(4) + 4 * rec
    assert kda.workspace_bytes(2, 65, 3, 64, 64) == tick + lst(12) + 2 * 6 * rec
    # long sequence: two buffers of as many chunks as fit in 1 GiB each, plus the carried state
    row = 32 * rec
    seg = (1 << 30) // row
    assert kda.workspace_bytes(1, 1 << 20, 32, 128, 128) == tick + lst(32 * seg) + 2 * seg * row + 32 * 128 * 128 * 4
    # unsupported or empty
    assert kda.workspace_bytes(1, 0, 1, 128, 128) == 0
    assert kda.workspace_bytes(1, 64, 1, 96, 128) == 0
    assert kda.workspace_bytes(0, 64, 1, 128, 128) == 0


def test_noalloc_rejects_beyond_its_scratch(lib):
    def call(B, H, hT, dk=128, dv=128):
        return lib.kda_chunk_fwd_noalloc(A, A, A, A, A, 1.0, None, A, hT, B, 64, H, dk, dv, None)
    # one chunk record of every (b, h) must fit in the 64 MiB array: B * H <= 903 with hT given
    assert call(1, 904, A) == kda.KDA_ERR_SCRATCH_LIMIT
    assert call(2, 452, A) == kda.KDA_ERR_SCRATCH_LIMIT
    # without hT the carried fp32 state shares the array
    assert call(1, 600, None) == kda.KDA_ERR_SCRATCH_LIMIT
    assert kda.status_string(kda.KDA_ERR_SCRATCH_LIMIT) == "KDA_ERR_SCRATCH_LIMIT"
    # the usual argument checks come first
    assert lib.kda_chunk_fwd_noalloc(None, A, A, A, A, 1.0, None, A, None, 1, 64, 1, 64, 64, None) == \
        kda.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd_noalloc(A, A, A, A, A, 1.0, None, A, None, 1, 64, 1, 96, 64, None) == \
        kda.KDA_ERR_UNSUPPORTED
    assert lib.kda_chunk_fwd_noalloc(MIS, A, A, A, A, 1.0, None, A, None, 1, 64, 1, 64, 64, None) == \
        kda.KDA_ERR_ALIGNMENT


FOUR = ctypes.c_void_p(0x10004)  # 4-byte aligned, not 8


def gdn_chunk(lib, q=A, k=A, v=A, g=A, beta=A, h0=None, out=A, hT=None, B=1, T=64, H=1, dk=64, dv=64):
    return lib.kda_gdn_chunk_fwd(q, k, v, g, beta, 1.0, h0, out, hT, B, T, H, dk, dv, None)


def gdn_decode(lib, q=A, k=A, v=A, g=A, beta=A, state=A, out=A, B=1, H=1, dk=64, dv=64):
    return lib.kda_gdn_decode_step(q, k, v, g, beta, 1.0, state, out, B, H, dk, dv, None)


@pytest.mark.parametrize("kw,code", [
    (dict(g=None), kda.KDA_ERR_INVALID_ARG),
    (dict(T=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(q=MIS), kda.KDA_ERR_ALIGNMENT),
    (dict(g=ODD), kda.KDA_ERR_ALIGNMENT),   # the scalar gate needs 4-byte alignment only
])
def test_gdn_chunk_fwd_rejects(lib, kw, code):
    assert gdn_chunk(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(g=None), kda.KDA_ERR_INVALID_ARG),
    (dict(dv=32), kda.KDA_ERR_UNSUPPORTED),
    (dict(state=MIS), kda.KDA_ERR_ALIGNMENT),
    (dict(g=ODD), kda.KDA_ERR_ALIGNMENT),
])
def test_gdn_decode_step_rejects(lib, kw, code):
    assert gdn_decode(lib, **kw) == code


def test_gate_alignment_rule_differs_by_form(lib):
    # a [B,T,H] scalar gate row is 4 bytes: a 4-byte-aligned gate passes validation
    # (T == 0, no h0/hT: validation only, nothing enqueued); the per-channel gate needs 16
    assert gdn_chunk(lib, g=FOUR, T=0) == kda.KDA_OK
    assert chunk(lib, g=FOUR, T=0) == kda.KDA_ERR_ALIGNMENT


def varlen(lib, q=A, k=A, v=A, g=A, beta=A, cu=A, N=2, h0=None, out=A, hT=None, T=100, H=1, dk=64, dv=64):
    return lib.kda_chunk_fwd_varlen(q, k, v, g, beta, 1.0, cu, N, h0, out, hT, T, H, dk, dv, None)


@pytest.mark.parametrize("kw,code", [
    (dict(cu=None), kda.KDA_ERR_INVALID_ARG),
    (dict(N=0), kda.KDA_ERR_INVALID_ARG),
    (dict(q=None), kda.KDA_ERR_INVALID_ARG),
    (dict(T=-1), kda.KDA_ERR_INVALID_ARG),
    (dict(H=0), kda.KDA_ERR_INVALID_ARG),
    (dict(dk=96), kda.KDA_ERR_UNSUPPORTED),
    (dict(cu=ODD), kda.KDA_ERR_ALIGNMENT),
    (dict(g=MIS), kda.KDA_ERR_ALIGNMENT),
    (dict(hT=MIS), kda.KDA_ERR_ALIGNMENT),
])
def test_varlen_rejects(lib, kw, code):
    assert varlen(lib, **kw) == code


def test_varlen_zero_tokens_accepts_null_inputs(lib):
    # T_total == 0 with no h0/hT: every sequence is empty, nothing to read or write
    assert varlen(lib, q=None, k=None, v=None, g=None, beta=None, out=None, T=0) == kda.KDA_OK


def test_varlen_workspace_bytes(lib):
    rec, tick = 74240, 256

    def r256(x):
        return (x + 255) // 256 * 256

    N, T, H = 3, 1000, 4
    cmax = T // 64 + N + 1  # chunks: at most one partial chunk per sequence
    assert kda.varlen_workspace_bytes(N, T, H, 128, 128) == \
        tick + r256(4 * H * cmax) + r256(4 * (2 * (N + 1) + cmax)) + cmax * H * rec
    assert kda.varlen_workspace_bytes(N, 0, H, 128, 128) == 0
    assert kda.varlen_workspace_bytes(0, 10, H, 128, 128) == 0


def test_raw_entry_points_validate_gate_scale(lib):
    def raw(c, **kw):
        a = dict(q=A, k=A, v=A, g=A, beta=A, h0=None, out=A, hT=None, B=1, T=64, H=1, dk=64, dv=64)
        a.update(kw)
        return lib.kda_chunk_fwd_raw(a["q"], a["k"], a["v"], a["g"], a["beta"], c, 1.0, a["h0"], a["out"], a["hT"],
                                     a["B"], a["T"], a["H"], a["dk"], a["dv"], None)
    assert raw(-0.5) == kda.KDA_ERR_INVALID_ARG
    assert raw(float("nan")) == kda.KDA_ERR_INVALID_ARG
    assert raw(0.5, q=None) == kda.KDA_ERR_INVALID_ARG
    assert raw(0.5, dk=96) == kda.KDA_ERR_UNSUPPORTED
    assert raw(0.5, k=MIS) == kda.KDA_ERR_ALIGNMENT
    assert lib.kda_decode_step_raw(A, A, A, A, A, -1.0, 1.0, A, A, 1, 1, 64, 64, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_decode_step_raw(A, A, A, A, A, 1.0, 1.0, None, A, 1, 1, 64, 64, None) == kda.KDA_ERR_INVALID_ARG


def test_backward_rejects(lib):
    def bwd(**kw):
        a = dict(q=A, k=A, v=A, g=A, beta=A, h0=None, dout=A, dhT=None, dq=A, dk=A, dv=A, dg=A, db=A, dh0=None,
                 B=1, T=64, H=1, dk_=64, dv_=64)
        a.update(kw)
        return lib.kda_chunk_bwd(a["q"], a["k"], a["v"], a["g"], a["beta"], 1.0, a["h0"], a["dout"], a["dhT"],
                                 a["dq"], a["dk"], a["dv"], a["dg"], a["db"], a["dh0"], a["B"], a["T"], a["H"],
                                 a["dk_"], a["dv_"], None)
    assert bwd(q=None) == kda.KDA_ERR_INVALID_ARG
    assert bwd(dg=None) == kda.KDA_ERR_INVALID_ARG
    assert bwd(B=0) == kda.KDA_ERR_INVALID_ARG
    assert bwd(dk_=96) == kda.KDA_ERR_UNSUPPORTED
    assert bwd(dq=MIS) == kda.KDA_ERR_ALIGNMENT
    assert bwd(db=ODD) == kda.KDA_ERR_ALIGNMENT
    # T == 0 with no dh0 wanted: nothing to do
    assert bwd(q=None, k=None, v=None, g=None, beta=None, dq=None, dk=None, dv=None, dg=None, db=None, T=0) == \
        kda.KDA_OK
    # a state every 64 tokens and a scratch of 16 states, then every token's p, per (b, h)
    assert lib.kda_chunk_bwd_workspace_bytes(2, 100, 3, 128, 64) == 2 * 3 * ((2 + 16) * 128 * 64 + 100 * 64) * 4


def test_debug_library_exports_the_same_symbols(lib):
    """libkda_debug.so (KDA_DEBUG: device-side index checks) is a separate build
    of the same sources with the same C ABI."""
    from gated_delta_rule_100_b200 import kda as k
    dbg = ctypes.CDLL(k.DEBUG_LIB_PATH)
    for name in declared_symbols():
        assert hasattr(dbg, name), name
    assert os.path.getsize(k.DEBUG_LIB_PATH) != os.path.getsize(k.LIB_PATH)
    assert kda.status_string(kda.KDA_ERR_BOUNDS) == "KDA_ERR_BOUNDS"
