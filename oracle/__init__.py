"""fp64 CPU oracle for the Kimi Delta Attention (KDA) forward pass.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, ``__graft_entry__.smoke()``
and the benchmark's CPU-baseline leg may import this package.  The CUDA
library never loads it and shares no code with it.

The recurrence (``kda_oracle.c``) is the combined update of "Kimi Linear's
Hybrid Linear Attention Architecture: A Technical Breakdown", section 3.3:
decay each key channel of the old state by alpha_t = exp(g_t), erase along
k_t with strength beta_t, write beta_t k_t v_t^T; then read
o_t = scale * S_t^T q_t.  The state is dk x dv, as in the update printed in
"Kimi Linear: How Moonshot AI Built a Hybrid Attention Architecture That
Beats Full Attention".

Every function takes and returns float64 numpy arrays in the library's
layouts: q, k, g [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H]; h0/hT [B,H,dk,dv];
out [B,T,H,dv].
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``libkda_oracle.so`` beside it (gcc, OpenMP).

    Plain -O2 without fast-math or FMA contraction, so each operation rounds
    as written.
    """
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    L = ctypes.c_long
    lib.kda_oracle_fwd.argtypes = [dp] * 6 + [ctypes.c_double, dp, dp, dp] + [L] * 5 + [ctypes.c_int]
    lib.kda_oracle_fwd.restype = ctypes.c_int
    lib.kda_oracle_bruteforce.argtypes = [dp] * 6 + [ctypes.c_double, dp, dp, dp] + [L] * 5
    lib.kda_oracle_bruteforce.restype = ctypes.c_int
    lib.kda_oracle_bwd.argtypes = [dp] * 6 + [ctypes.c_double, dp, dp, dp] + [dp] * 7 + [L] * 5 + [ctypes.c_int]
    lib.kda_oracle_bwd.restype = ctypes.c_int
    lib.kda_oracle_max_threads.restype = ctypes.c_int
    return lib


def _load(lib=None):
    """The default oracle library, or ``lib`` when a caller passes its own build."""
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def load_library(path: str):
    """Bind another build of ``kda_oracle.c`` (the tests use this for planted mistakes)."""
    return _bind(path)


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _prep(q, k, v, g, beta, h0, erase, write):
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != (B, T, H, dk) or g.shape != (B, T, H, dk) or v.shape != (B, T, H, dv):
        raise ValueError("q, k, g must be [B,T,H,dk] and v [B,T,H,dv]")
    if beta is not None:
        beta = _f64(beta)
        if beta.shape != (B, T, H):
            raise ValueError("beta must be [B,T,H]")
    e = beta if erase is None else _f64(erase)
    w = beta if write is None else _f64(write)
    if e is None or w is None:
        raise ValueError("beta, or both erase and write weights, must be given")
    if e.shape != (B, T, H) or w.shape != (B, T, H):
        raise ValueError("erase/write weights must be [B,T,H]")
    if h0 is not None:
        h0 = _f64(h0)
        if h0.shape != (B, H, dk, dv):
            raise ValueError("h0 must be [B,H,dk,dv]")
    return q, k, v, g, e, w, h0, (B, T, H, dk, dv)


def kda_fwd(q, k, v, g, beta, scale, h0=None, *, erase=None, write=None,
            threads: int | None = None, lib=None):
    """Run the recurrence token by token.  Returns (out, hT), both float64.

    ``erase`` / ``write`` override beta on the erase term and on the write
    term separately (KDA uses the same beta for both); they let the tests
    reach the gated linear-attention special cases.
    """
    q, k, v, g, e, w, h0, (B, T, H, dk, dv) = _prep(q, k, v, g, beta, h0, erase, write)
    out = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dk, dv))
    lib = _load(lib)
    nt = int(lib.kda_oracle_max_threads()) if threads is None else int(threads)
    rc = lib.kda_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(e), _ptr(w),
                                float(scale), _ptr(h0), _ptr(out), _ptr(hT),
                                B, T, H, dk, dv, nt)
    if rc != 0:
        raise RuntimeError("kda_oracle_fwd failed")
    return out, hT


def kda_bruteforce(q, k, v, g, beta, scale, h0=None, *, erase=None, write=None, lib=None):
    """Same recurrence through explicit dk x dk transition matrices (small T only)."""
    q, k, v, g, e, w, h0, (B, T, H, dk, dv) = _prep(q, k, v, g, beta, h0, erase, write)
    out = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dk, dv))
    rc = _load(lib).kda_oracle_bruteforce(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(e), _ptr(w),
                                       float(scale), _ptr(h0), _ptr(out), _ptr(hT),
                                       B, T, H, dk, dv)
    if rc != 0:
        raise RuntimeError("kda_oracle_bruteforce failed")
    return out, hT


def kda_bwd(q, k, v, g, beta, scale, h0=None, dout=None, dhT=None, *, erase=None, write=None,
            threads: int | None = None, lib=None):
    """Gradients of sum(dout * out) + sum(dhT * hT) with respect to the inputs of
    ``kda_fwd``, by reverse-mode differentiation of the token loop.  Returns a
    dict with dq, dk, dv, dg, dbeta (= derase + dwrite), derase, dwrite, dh0
    (float64, the inputs' layouts).  Keeps every state of a (b, h): small T only."""
    q, k, v, g, e, w, h0, (B, T, H, dk, dv) = _prep(q, k, v, g, beta, h0, erase, write)
    dout = None if dout is None else _f64(dout)
    dhT = None if dhT is None else _f64(dhT)
    if dout is not None and dout.shape != (B, T, H, dv):
        raise ValueError("dout must be [B,T,H,dv]")
    if dhT is not None and dhT.shape != (B, H, dk, dv):
        raise ValueError("dhT must be [B,H,dk,dv]")
    r = {n: np.zeros((B, T, H, dk)) for n in ("dq", "dk", "dg")}
    r["dv"] = np.zeros((B, T, H, dv))
    r["derase"] = np.zeros((B, T, H))
    r["dwrite"] = np.zeros((B, T, H))
    r["dh0"] = np.zeros((B, H, dk, dv))
    lib = _load(lib)
    nt = int(lib.kda_oracle_max_threads()) if threads is None else int(threads)
    rc = lib.kda_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(e), _ptr(w), float(scale), _ptr(h0),
                            _ptr(dout), _ptr(dhT), _ptr(r["dq"]), _ptr(r["dk"]), _ptr(r["dv"]), _ptr(r["dg"]),
                            _ptr(r["derase"]), _ptr(r["dwrite"]), _ptr(r["dh0"]), B, T, H, dk, dv, nt)
    if rc != 0:
        raise RuntimeError("kda_oracle_bwd failed")
    r["dbeta"] = r["derase"] + r["dwrite"]
    return r


def kda_decode_step(q, k, v, g, beta, scale, state, threads: int | None = None, lib=None):
    """One recurrent step for every (b, h): inputs [B,H,*], beta [B,H], state [B,H,dk,dv].

    Returns (out [B,H,dv], new_state).  It is ``kda_fwd`` with T = 1 and the
    carried state as h0.
    """
    q, k, v, g = (_f64(x)[:, None] for x in (q, k, v, g))
    beta = _f64(beta)[:, None]
    out, hT = kda_fwd(q, k, v, g, beta, scale, h0=state, threads=threads, lib=lib)
    return out[:, 0], hT
