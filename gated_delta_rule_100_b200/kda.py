"""Python binding of libkda (ctypes).  Argument marshalling only: every step of
the computation runs in the library's CUDA kernels.

The entry points mirror ``include/kda.h``:

* ``chunk_fwd``   -> ``kda_chunk_fwd``   (chunkwise prefill)
* ``chunk_fwd_noalloc`` -> ``kda_chunk_fwd_noalloc`` (the same prefill over a fixed
  scratch array: no device allocation)
* ``chunk_fwd_varlen`` -> ``kda_chunk_fwd_varlen`` (packed batch of sequences, cu_seqlens)
* ``decode_step`` -> ``kda_decode_step`` (one recurrent step, state in place)
* ``chunk_fwd_raw`` / ``decode_step_raw`` -> ``kda_chunk_fwd_raw`` / ``kda_decode_step_raw``
  (raw projections in: the gate prologue and the q/k normalisation run in the kernels)
* ``stream_status`` -> ``kda_stream_status``
* ``workspace_bytes`` / ``release_workspace`` -> ``kda_chunk_fwd_workspace_bytes`` /
  ``kda_release_workspace``

* ``chunk_fwd_host`` -> ``kda_chunk_fwd_host`` (the prefill on host tensors, pinned for
  overlap: the library streams pieces of the token axis up, through the prefill and back)

If ``libkda.so`` is missing the calls raise; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")
DEBUG_LIB_PATH = os.path.join(_HERE, "libkda_debug.so")

(KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_ALIGNMENT, KDA_ERR_CUDA, KDA_ERR_TIMEOUT,
 KDA_ERR_SCRATCH_LIMIT, KDA_ERR_BOUNDS) = range(8)
EXPORTED = ("kda_chunk_fwd", "kda_chunk_fwd_noalloc", "kda_chunk_fwd_host", "kda_chunk_fwd_host_debug_piece", "kda_chunk_fwd_varlen", "kda_decode_step",
            "kda_gdn_chunk_fwd", "kda_gdn_decode_step", "kda_chunk_fwd_raw", "kda_decode_step_raw",
            "kda_chunk_bwd", "kda_chunk_bwd_workspace_bytes",
            "kda_chunk_fwd_workspace_bytes", "kda_chunk_fwd_varlen_workspace_bytes", "kda_release_workspace",
            "kda_status_string", "kda_stream_status", "kda_chunk_fwd_debug_wait_limit",
            "kda_chunk_fwd_debug_inject_timeout", "kda_chunk_fwd_debug_force_exact", "kda_chunk_fwd_debug_block_refs", "kda_chunk_fwd_debug_record_cap", "kda_chunk_fwd_debug_parts",
            "kda_debug_kernel_timing", "kda_debug_kernel_times", "kda_debug_kernel_launches",
            "kda_abi_version")

_lib = None          # the library the calls below go through
_libs = {}           # path -> loaded library


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load():
    """The library the binding's calls go through: libkda.so (built in-tree by
    ``gated_delta_rule_100_b200.build``) unless ``use_debug_library(True)``."""
    global _lib
    if _lib is None:
        _lib = _open(LIB_PATH)
    return _lib


def use_debug_library(enable: bool) -> None:
    """Route every call through libkda_debug.so (device-side index checks that
    report KDA_ERR_BOUNDS) or back through libkda.so.  The two libraries have
    separate device state (status word, workspace)."""
    global _lib
    _lib = _open(DEBUG_LIB_PATH if enable else LIB_PATH)


def _open(path):
    if path in _libs:
        return _libs[path]
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m gated_delta_rule_100_b200.build`")
    lib = ctypes.CDLL(path)
    vp, fp, i, f = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp, i, i, i, i, i, vp]
    lib.kda_chunk_fwd.restype = i
    lib.kda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp, i, i, i, i, i, vp]
    lib.kda_chunk_fwd_noalloc.restype = i
    lib.kda_chunk_fwd_host.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp, i, i, i, i, i, vp]
    lib.kda_chunk_fwd_host.restype = i
    lib.kda_chunk_fwd_host_debug_piece.argtypes = [i]
    lib.kda_chunk_fwd_host_debug_piece.restype = None
    lib.kda_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp, vp, vp, vp, fp, fp, fp, i, i, i, i, i, vp]
    lib.kda_chunk_bwd.restype = i
    lib.kda_chunk_bwd_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.kda_chunk_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.kda_chunk_fwd_raw.argtypes = [vp, vp, vp, fp, fp, f, f, fp, vp, fp, i, i, i, i, i, vp]
    lib.kda_chunk_fwd_raw.restype = i
    lib.kda_decode_step_raw.argtypes = [vp, vp, vp, fp, fp, f, f, fp, vp, i, i, i, i, vp]
    lib.kda_decode_step_raw.restype = i
    lib.kda_chunk_fwd_varlen.argtypes = [vp, vp, vp, fp, fp, f, vp, i, fp, vp, fp, i, i, i, i, vp]
    lib.kda_chunk_fwd_varlen.restype = i
    lib.kda_chunk_fwd_varlen_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.kda_chunk_fwd_varlen_workspace_bytes.restype = ctypes.c_size_t
    lib.kda_decode_step.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, i, i, i, i, vp]
    lib.kda_decode_step.restype = i
    lib.kda_gdn_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, fp, i, i, i, i, i, vp]
    lib.kda_gdn_chunk_fwd.restype = i
    lib.kda_gdn_decode_step.argtypes = [vp, vp, vp, fp, fp, f, fp, vp, i, i, i, i, vp]
    lib.kda_gdn_decode_step.restype = i
    lib.kda_chunk_fwd_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.kda_chunk_fwd_workspace_bytes.restype = ctypes.c_size_t
    lib.kda_release_workspace.argtypes = []
    lib.kda_release_workspace.restype = i
    lib.kda_status_string.argtypes = [i]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_stream_status.argtypes = [vp]
    lib.kda_stream_status.restype = i
    lib.kda_chunk_fwd_debug_wait_limit.argtypes = [ctypes.c_ulonglong]
    lib.kda_chunk_fwd_debug_wait_limit.restype = None
    lib.kda_chunk_fwd_debug_inject_timeout.argtypes = [ctypes.c_ulonglong]
    lib.kda_chunk_fwd_debug_inject_timeout.restype = None
    lib.kda_chunk_fwd_debug_parts.argtypes = [i]
    lib.kda_chunk_fwd_debug_parts.restype = None
    lib.kda_chunk_fwd_debug_record_cap.argtypes = [ctypes.c_ulonglong]
    lib.kda_chunk_fwd_debug_record_cap.restype = None
    lib.kda_chunk_fwd_debug_force_exact.argtypes = [i]
    lib.kda_chunk_fwd_debug_force_exact.restype = None
    lib.kda_chunk_fwd_debug_block_refs.argtypes = [i]
    lib.kda_chunk_fwd_debug_block_refs.restype = None
    lib.kda_debug_kernel_timing.argtypes = [i]
    lib.kda_debug_kernel_timing.restype = None
    lib.kda_debug_kernel_times.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong), i]
    lib.kda_debug_kernel_times.restype = i
    ll = ctypes.POINTER(ctypes.c_longlong)
    lib.kda_debug_kernel_launches.argtypes = [ctypes.POINTER(ctypes.c_int), ll, ll, i, ctypes.POINTER(ctypes.c_int)]
    lib.kda_debug_kernel_launches.restype = i
    lib.kda_abi_version.restype = i
    _libs[path] = lib
    return lib


def status_string(status: int) -> str:
    return load().kda_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t, name, dtype, shape):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def chunk_fwd(q, k, v, g, beta, scale, h0=None, *, out=None, hT=None, final_state=True, stream=None):
    """Chunkwise prefill.  q, k [B,T,H,dk] bf16; v [B,T,H,dv] bf16; g [B,T,H,dk] fp32;
    beta [B,T,H] fp32; h0 [B,H,dk,dv] fp32 or None.  Returns (out, hT); hT is None
    when ``final_state`` is False and no ``hT`` buffer was given."""
    return _prefill("kda_chunk_fwd", False, q, k, v, g, beta, scale, h0, out, hT, final_state, stream)


def gdn_chunk_fwd(q, k, v, g, beta, scale, h0=None, *, out=None, hT=None, final_state=True, stream=None):
    """Scalar-gate (Gated DeltaNet) prefill: as ``chunk_fwd`` with g [B,T,H] fp32, one
    log-decay per token and head shared by every key channel."""
    return _prefill("kda_gdn_chunk_fwd", True, q, k, v, g, beta, scale, h0, out, hT, final_state, stream)


def _prefill(symbol, scalar_gate, q, k, v, g, beta, scale, h0, out, hT, final_state, stream):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", torch.bfloat16, (B, T, H, dk))
    _check(k, "k", torch.bfloat16, (B, T, H, dk))
    _check(v, "v", torch.bfloat16, (B, T, H, dv))
    _check(g, "g", torch.float32, (B, T, H) if scalar_gate else (B, T, H, dk))
    _check(beta, "beta", torch.float32, (B, T, H))
    if h0 is not None:
        _check(h0, "h0", torch.float32, (B, H, dk, dv))
    if out is None:
        out = torch.empty((B, T, H, dv), device=q.device, dtype=torch.bfloat16)
    _check(out, "out", torch.bfloat16, (B, T, H, dv))
    if hT is None and final_state:
        hT = torch.empty((B, H, dk, dv), device=q.device, dtype=torch.float32)
    if hT is not None:
        _check(hT, "hT", torch.float32, (B, H, dk, dv))
    rc = getattr(load(), symbol)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                 _ptr(h0), _ptr(out), _ptr(hT), B, T, H, dk, dv, _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, symbol)
    return out, hT


def chunk_bwd(q, k, v, g, beta, scale, h0=None, dout=None, dhT=None, *, want_dh0=True, stream=None):
    """Backward of ``chunk_fwd``: gradients of L given dL/dout (bf16 [B,T,H,dv]) and
    dL/dhT (fp32 [B,H,dk,dv]); either may be None (zero).  Returns a dict with dq, dk,
    dv (bf16), dg, dbeta and dh0 (fp32; None when ``want_dh0`` is False)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", torch.bfloat16, (B, T, H, dk))
    _check(k, "k", torch.bfloat16, (B, T, H, dk))
    _check(v, "v", torch.bfloat16, (B, T, H, dv))
    _check(g, "g", torch.float32, (B, T, H, dk))
    _check(beta, "beta", torch.float32, (B, T, H))
    if h0 is not None:
        _check(h0, "h0", torch.float32, (B, H, dk, dv))
    if dout is not None:
        _check(dout, "dout", torch.bfloat16, (B, T, H, dv))
    if dhT is not None:
        _check(dhT, "dhT", torch.float32, (B, H, dk, dv))
    z = dict(device=q.device)
    r = dict(dq=torch.empty((B, T, H, dk), dtype=torch.bfloat16, **z),
             dk=torch.empty((B, T, H, dk), dtype=torch.bfloat16, **z),
             dv=torch.empty((B, T, H, dv), dtype=torch.bfloat16, **z),
             dg=torch.empty((B, T, H, dk), dtype=torch.float32, **z),
             dbeta=torch.empty((B, T, H), dtype=torch.float32, **z),
             dh0=torch.empty((B, H, dk, dv), dtype=torch.float32, **z) if want_dh0 else None)
    rc = load().kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(h0), _ptr(dout),
                              _ptr(dhT), _ptr(r["dq"]), _ptr(r["dk"]), _ptr(r["dv"]), _ptr(r["dg"]), _ptr(r["dbeta"]),
                              _ptr(r["dh0"]), B, T, H, dk, dv, _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_bwd")
    return r


def chunk_fwd_raw(q, k, v, g_raw, beta_raw, gate_c, scale, h0=None, *, out=None, hT=None, final_state=True,
                  stream=None):
    """Prefill from raw projections: g = -gate_c softplus(g_raw), beta = sigmoid(beta_raw),
    q and k L2-normalised, all inside the kernels.  Shapes and dtypes as ``chunk_fwd``."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", torch.bfloat16, (B, T, H, dk))
    _check(k, "k", torch.bfloat16, (B, T, H, dk))
    _check(v, "v", torch.bfloat16, (B, T, H, dv))
    _check(g_raw, "g_raw", torch.float32, (B, T, H, dk))
    _check(beta_raw, "beta_raw", torch.float32, (B, T, H))
    if h0 is not None:
        _check(h0, "h0", torch.float32, (B, H, dk, dv))
    if out is None:
        out = torch.empty((B, T, H, dv), device=q.device, dtype=torch.bfloat16)
    _check(out, "out", torch.bfloat16, (B, T, H, dv))
    if hT is None and final_state:
        hT = torch.empty((B, H, dk, dv), device=q.device, dtype=torch.float32)
    if hT is not None:
        _check(hT, "hT", torch.float32, (B, H, dk, dv))
    rc = load().kda_chunk_fwd_raw(_ptr(q), _ptr(k), _ptr(v), _ptr(g_raw), _ptr(beta_raw), float(gate_c),
                                  float(scale), _ptr(h0), _ptr(out), _ptr(hT), B, T, H, dk, dv, _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_raw")
    return out, hT


def decode_step_raw(q, k, v, g_raw, beta_raw, gate_c, scale, state, *, out=None, stream=None):
    """One recurrent step from raw projections (see ``chunk_fwd_raw``); shapes as ``decode_step``."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", torch.bfloat16, (B, H, dk))
    _check(k, "k", torch.bfloat16, (B, H, dk))
    _check(v, "v", torch.bfloat16, (B, H, dv))
    _check(g_raw, "g_raw", torch.float32, (B, H, dk))
    _check(beta_raw, "beta_raw", torch.float32, (B, H))
    _check(state, "state", torch.float32, (B, H, dk, dv))
    if out is None:
        out = torch.empty((B, H, dv), device=q.device, dtype=torch.bfloat16)
    _check(out, "out", torch.bfloat16, (B, H, dv))
    rc = load().kda_decode_step_raw(_ptr(q), _ptr(k), _ptr(v), _ptr(g_raw), _ptr(beta_raw), float(gate_c),
                                    float(scale), _ptr(state), _ptr(out), B, H, dk, dv, _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_decode_step_raw")
    return out


def chunk_fwd_noalloc(q, k, v, g, beta, scale, h0=None, *, out, hT=None, stream=None):
    """``chunk_fwd`` through ``kda_chunk_fwd_noalloc``: the caller passes ``out``
    (and ``hT`` unless the final state is not wanted); the library allocates
    nothing.  Returns (out, hT)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", torch.bfloat16, (B, T, H, dk))
    _check(k, "k", torch.bfloat16, (B, T, H, dk))
    _check(v, "v", torch.bfloat16, (B, T, H, dv))
    _check(g, "g", torch.float32, (B, T, H, dk))
    _check(beta, "beta", torch.float32, (B, T, H))
    if h0 is not None:
        _check(h0, "h0", torch.float32, (B, H, dk, dv))
    _check(out, "out", torch.bfloat16, (B, T, H, dv))
    if hT is not None:
        _check(hT, "hT", torch.float32, (B, H, dk, dv))
    rc = load().kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                      _ptr(h0), _ptr(out), _ptr(hT), B, T, H, dk, dv, _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_noalloc")
    return out, hT


def chunk_fwd_varlen(q, k, v, g, beta, scale, cu_seqlens, h0=None, *, out=None, hT=None, final_state=True,
                     stream=None):
    """Prefill of a packed batch.  q, k [T_total,H,dk] bf16; v [T_total,H,dv] bf16;
    g [T_total,H,dk] fp32; beta [T_total,H] fp32; cu_seqlens int32 [N+1] on the
    device; h0 [N,H,dk,dv] fp32 or None.  Returns (out [T_total,H,dv], hT [N,H,dk,dv]);
    hT is None when ``final_state`` is False and no ``hT`` buffer was given."""
    T, H, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", torch.bfloat16, (T, H, dk))
    _check(k, "k", torch.bfloat16, (T, H, dk))
    _check(v, "v", torch.bfloat16, (T, H, dv))
    _check(g, "g", torch.float32, (T, H, dk))
    _check(beta, "beta", torch.float32, (T, H))
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be a 1-D tensor of N + 1 >= 2 offsets")
    N = cu_seqlens.numel() - 1
    _check(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,))
    if h0 is not None:
        _check(h0, "h0", torch.float32, (N, H, dk, dv))
    if out is None:
        out = torch.empty((T, H, dv), device=q.device, dtype=torch.bfloat16)
    _check(out, "out", torch.bfloat16, (T, H, dv))
    if hT is None and final_state:
        hT = torch.empty((N, H, dk, dv), device=q.device, dtype=torch.float32)
    if hT is not None:
        _check(hT, "hT", torch.float32, (N, H, dk, dv))
    rc = load().kda_chunk_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                     _ptr(cu_seqlens), N, _ptr(h0), _ptr(out), _ptr(hT), T, H, dk, dv,
                                     _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_varlen")
    return out, hT


def varlen_workspace_bytes(N: int, T_total: int, H: int, dk: int, dv: int) -> int:
    """Device memory ``chunk_fwd_varlen`` holds for these sizes (0 when unsupported)."""
    return int(load().kda_chunk_fwd_varlen_workspace_bytes(int(N), int(T_total), int(H), int(dk), int(dv)))


def set_parts(parts: int) -> None:
    """Test hook: parts of the two-level pass (0 = automatic, 1 = off, P >= 3 = forced)."""
    load().kda_chunk_fwd_debug_parts(int(parts))


def set_record_cap(nbytes: int) -> None:
    """Test hook: cap the chunk records the prefill workspace holds (0 = default)."""
    load().kda_chunk_fwd_debug_record_cap(int(nbytes))


def decode_step(q, k, v, g, beta, scale, state, *, out=None, stream=None):
    """One recurrent step.  q, k [B,H,dk] bf16; v [B,H,dv] bf16; g [B,H,dk] fp32;
    beta [B,H] fp32; state [B,H,dk,dv] fp32 (updated in place).  Returns out [B,H,dv] bf16."""
    return _decode("kda_decode_step", False, q, k, v, g, beta, scale, state, out, stream)


def gdn_decode_step(q, k, v, g, beta, scale, state, *, out=None, stream=None):
    """Scalar-gate (Gated DeltaNet) decode step: as ``decode_step`` with g [B,H] fp32."""
    return _decode("kda_gdn_decode_step", True, q, k, v, g, beta, scale, state, out, stream)


def _decode(symbol, scalar_gate, q, k, v, g, beta, scale, state, out, stream):
    B, H, dk = q.shape
    dv = v.shape[-1]
    _check(q, "q", torch.bfloat16, (B, H, dk))
    _check(k, "k", torch.bfloat16, (B, H, dk))
    _check(v, "v", torch.bfloat16, (B, H, dv))
    _check(g, "g", torch.float32, (B, H) if scalar_gate else (B, H, dk))
    _check(beta, "beta", torch.float32, (B, H))
    _check(state, "state", torch.float32, (B, H, dk, dv))
    if out is None:
        out = torch.empty((B, H, dv), device=q.device, dtype=torch.bfloat16)
    _check(out, "out", torch.bfloat16, (B, H, dv))
    rc = getattr(load(), symbol)(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                                 _ptr(state), _ptr(out), B, H, dk, dv, _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, symbol)
    return out


def workspace_bytes(B: int, T: int, H: int, dk: int, dv: int) -> int:
    """Device memory ``chunk_fwd`` holds for these sizes (0 when unsupported)."""
    return int(load().kda_chunk_fwd_workspace_bytes(int(B), int(T), int(H), int(dk), int(dv)))


def release_workspace() -> None:
    """Free the current device's prefill workspace (synchronises the device)."""
    rc = load().kda_release_workspace()
    if rc != KDA_OK:
        raise KdaError(rc, "kda_release_workspace")


def stream_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(load().kda_stream_status(_stream(stream)))


def set_wait_limit(polls: int) -> None:
    """Test hook: polls a device-side wait makes before giving up (0 = default)."""
    load().kda_chunk_fwd_debug_wait_limit(int(polls))


def inject_timeout(polls: int) -> None:
    """Test hook: nonzero makes each prefill CTA first wait on a barrier nothing
    signals (at most ``polls`` polls) and take its timeout path; 0 = off."""
    load().kda_chunk_fwd_debug_inject_timeout(int(polls))


def force_exact(enable: bool) -> None:
    """Test hook: every prefill chunk takes the exact path (see ``kda.h``)."""
    load().kda_chunk_fwd_debug_force_exact(1 if enable else 0)


def block_refs(enable: bool) -> None:
    """Test hook: every prefill chunk is formed with its 16-token block
    references, mild decay or not (see ``kda.h``)."""
    load().kda_chunk_fwd_debug_block_refs(1 if enable else 0)


KERNEL_KINDS = ("prep", "chain", "exact", "fixup", "bwd")


def kernel_timing(enable: bool) -> None:
    """Measurement hook: every prefill and backward launch stamps its first CTA's
    start and last CTA's end (device globaltimer)."""
    load().kda_debug_kernel_timing(1 if enable else 0)


def kernel_times() -> dict:
    """{kind: (ms summed, launches)} of the launches timed since the last call."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_longlong * n)()
    rc = load().kda_debug_kernel_times(ms, cnt, n)
    if rc != KDA_OK:
        raise KdaError(rc, "kda_debug_kernel_times")
    return {k: (ms[i], int(cnt[i])) for i, k in enumerate(KERNEL_KINDS)}


def kernel_launches(cap: int = 8192) -> list:
    """[(kind, start_ms, end_ms)] of the launches timed since the last read, in launch
    order, times relative to the first start (end < start: no stamp)."""
    kind = (ctypes.c_int * cap)()
    st, en = (ctypes.c_longlong * cap)(), (ctypes.c_longlong * cap)()
    cnt = ctypes.c_int(0)
    rc = load().kda_debug_kernel_launches(kind, st, en, cap, ctypes.byref(cnt))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_debug_kernel_launches")
    n = cnt.value
    t0 = min((st[i] for i in range(n) if en[i] >= st[i]), default=0)
    return [(KERNEL_KINDS[kind[i]] if 0 <= kind[i] < len(KERNEL_KINDS) else kind[i],
             (st[i] - t0) * 1e-6, (en[i] - t0) * 1e-6) for i in range(n)]


def _check_host(t, name, dtype, shape):
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def chunk_fwd_host(q, k, v, g, beta, scale, h0=None, *, out, hT=None, stream=None):
    """``kda_chunk_fwd_host``: the prefill on HOST tensors (pinned, for overlapped copies),
    shapes and dtypes as ``chunk_fwd``; writes ``out`` (and ``hT`` when given) once
    ``stream`` reaches the end of the call's work.  Returns (bytes_h2d, bytes_d2h)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    _check_host(q, "q", torch.bfloat16, (B, T, H, dk))
    _check_host(k, "k", torch.bfloat16, (B, T, H, dk))
    _check_host(v, "v", torch.bfloat16, (B, T, H, dv))
    _check_host(g, "g", torch.float32, (B, T, H, dk))
    _check_host(beta, "beta", torch.float32, (B, T, H))
    _check_host(out, "out", torch.bfloat16, (B, T, H, dv))
    if h0 is not None:
        _check_host(h0, "h0", torch.float32, (B, H, dk, dv))
    if hT is not None:
        _check_host(hT, "hT", torch.float32, (B, H, dk, dv))
    rc = load().kda_chunk_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(h0),
                                   _ptr(out), _ptr(hT), B, T, H, dk, dv, _stream(stream))
    if rc != KDA_OK:
        raise KdaError(rc, "kda_chunk_fwd_host")
    nin = sum(t.numel() * t.element_size() for t in (q, k, v, g, beta, h0) if t is not None)
    nout = sum(t.numel() * t.element_size() for t in (out, hT) if t is not None)
    return nin, nout


def set_host_piece(tokens: int) -> None:
    """Test hook: pieces of ``tokens`` tokens for ``chunk_fwd_host`` (0 = automatic)."""
    load().kda_chunk_fwd_host_debug_piece(int(tokens))
