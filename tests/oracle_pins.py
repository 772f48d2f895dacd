"""Checks that pin the fp64 oracle to facts fixed by the pages and by algebra.

Each ``pin_*`` function runs the oracle (``lib`` selects a build, so the
planted-mistake tests can reuse them) and returns the largest deviation it
found from a value derived independently of the oracle's code: a hand
worked example, a closed form, a textbook special case computed with numpy
matrix products, an algebraic identity, or the explicit transition-matrix
product.  ``PIN_TOL`` gives the bound each must stay under.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kda_worked_examples.json")


def rand_case(rng, B=2, T=23, H=3, dk=5, dv=7, decay=0.3, h0=True, unit_k=True):
    """Random fp64 inputs with g <= 0, beta in (0, 1), unit-norm keys."""
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    g = -decay * np.log1p(np.exp(rng.standard_normal((B, T, H, dk))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    s0 = 0.5 * rng.standard_normal((B, H, dk, dv)) if h0 else None
    return q, k, v, g, beta, s0


def _maxabs(a, b):
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) if np.size(a) else 0.0


def pin_worked_examples(lib=None):
    """Hand-derived values in tests/golden/kda_worked_examples.json."""
    spec = json.load(open(GOLDEN))
    worst = 0.0
    for ex in spec["examples"]:
        T, dk, dv = ex["T"], ex["dk"], ex["dv"]

        def arr(x, shape):
            vals = [[math.log(0.5) if e == "log_half" else float(e) for e in row] for row in x]
            return np.array(vals, dtype=np.float64).reshape(shape)

        q = arr(ex["q"], (1, T, 1, dk))
        k = arr(ex["k"], (1, T, 1, dk))
        v = arr(ex["v"], (1, T, 1, dv))
        g = arr(ex["g"], (1, T, 1, dk))
        beta = np.array(ex["beta"], dtype=np.float64).reshape(1, T, 1)
        h0 = arr(ex["h0"], (1, 1, dk, dv))
        scales = ex["scale"] if isinstance(ex["scale"], list) else [ex["scale"]]
        for sc in scales:
            want = ex["out_by_scale"][repr(float(sc))] if "out_by_scale" in ex else ex["out"]
            want = np.array(want, dtype=np.float64).reshape(1, T, 1, dv)
            for fn in (oracle.kda_fwd, oracle.kda_bruteforce):
                out, hT = fn(q, k, v, g, beta, sc, h0, lib=lib)
                worst = max(worst, _maxabs(out, want),
                            _maxabs(hT, np.array(ex["hT"], dtype=np.float64).reshape(1, 1, dk, dv)))
    return worst


def pin_beta_zero_closed_form(lib=None, seed=1):
    """beta = 0: no erase and no write, so S_t = Diag(exp(Gamma_t)) h0 with
    Gamma_t the running sum of g, and o_t = scale * h0^T (exp(Gamma_t) * q_t)."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng)
    beta = np.zeros_like(beta)
    scale = 0.37
    out, hT = oracle.kda_fwd(q, k, v, g, beta, scale, h0, lib=lib)
    Gam = np.cumsum(g, axis=1)                                     # [B,T,H,dk]
    want = scale * np.einsum("bthc,bhcd->bthd", np.exp(Gam) * q, h0)
    want_hT = np.exp(Gam[:, -1])[..., None] * h0
    return max(_maxabs(out, want), _maxabs(hT, want_hT))


def pin_gated_linear_attention(lib=None, seed=2):
    """Erase weight 0, write weight 1: S_t = S_{t-1} Diag-decayed + k_t v_t^T (the
    diagonal-decay form of section 3.2 of the Baidu breakdown).  Unrolled:
    S_t = Diag(e^{Gamma_t}) h0 + sum_{j<=t} Diag(e^{Gamma_t - Gamma_j}) k_j v_j^T,
    evaluated as an O(T^2) double sum."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=17)
    zeros, ones = np.zeros_like(beta), np.ones_like(beta)
    scale = 0.8
    out, hT = oracle.kda_fwd(q, k, v, g, None, scale, h0, erase=zeros, write=ones, lib=lib)
    B, T, H, dk = q.shape
    Gam = np.cumsum(g, axis=1)
    want = np.zeros_like(out)
    for t in range(T):
        S = np.exp(Gam[:, t])[..., None] * h0                      # [B,H,dk,dv]
        for j in range(t + 1):
            dec = np.exp(Gam[:, t] - Gam[:, j])                    # [B,H,dk]
            S = S + (dec * k[:, j])[..., None] * v[:, j][:, :, None, :]
        want[:, t] = scale * np.einsum("bhc,bhcd->bhd", q[:, t], S)
        if t == T - 1:
            want_hT = S
    return max(_maxabs(out, want), _maxabs(hT, want_hT))


def pin_linear_attention(lib=None, seed=3):
    """alpha = 1, erase 0, write 1: plain linear attention S_t = S_{t-1} + k_t v_t^T
    (section 3.1 of the Baidu breakdown), i.e. causal (Q K^T) V plus the h0 read."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=19)
    g = np.zeros_like(g)
    scale = 1.3
    out, hT = oracle.kda_fwd(q, k, v, g, None, scale, h0,
                             erase=np.zeros_like(beta), write=np.ones_like(beta), lib=lib)
    B, T, H, dk = q.shape
    mask = np.tril(np.ones((T, T)))
    scores = np.einsum("bthc,bshc->bhts", q, k) * mask             # [B,H,T,T]
    want = scale * (np.einsum("bhts,bshd->bthd", scores, v)
                    + np.einsum("bthc,bhcd->bthd", q, h0))
    want_hT = h0 + np.einsum("bshc,bshd->bhcd", k, v)
    return max(_maxabs(out, want), _maxabs(hT, want_hT))


def pin_write_then_read(lib=None, seed=4):
    """beta = 1, unit k, any alpha: k^T (I - k k^T) = 0, so S_t^T k_t = v_t.
    With q_t = k_t and scale s the readout is exactly s * v_t at every step."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=29, decay=1.0)
    beta = np.ones_like(beta)
    out, _ = oracle.kda_fwd(k, k, v, g, beta, 0.25, h0, lib=lib)
    return _maxabs(out, 0.25 * v)


def pin_write_read_identity(lib=None, seed=5):
    """General beta, non-unit k: S_t^T k_t = (1 - b|k|^2)(D_t S_{t-1})^T k_t + b|k|^2 v_t.
    Checked step by step, carrying the state between one-token calls."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=9, unit_k=False)
    k = k * 0.7
    S = h0
    worst = 0.0
    for t in range(q.shape[1]):
        sl = slice(t, t + 1)
        out, S_new = oracle.kda_fwd(k[:, sl], k[:, sl], v[:, sl], g[:, sl], beta[:, sl], 1.0, S, lib=lib)
        kk = np.sum(k[:, t] ** 2, axis=-1)                          # [B,H]
        b = beta[:, t]
        DS = np.exp(g[:, t])[..., None] * S
        lhs = np.einsum("bhcd,bhc->bhd", S_new, k[:, t])
        rhs = ((1 - b * kk)[..., None] * np.einsum("bhcd,bhc->bhd", DS, k[:, t])
               + (b * kk)[..., None] * v[:, t])
        worst = max(worst, _maxabs(lhs, rhs), _maxabs(out[:, 0], lhs))
        S = S_new
    return worst


def pin_bruteforce(lib=None, seed=6, T=16):
    """Explicit transition matrices M_t = (I - b k k^T) Diag(alpha_t), dk != dv."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=T, dk=6, dv=4, unit_k=False)
    a = oracle.kda_fwd(q, k, v, g, beta, 0.6, h0, lib=lib)
    b = oracle.kda_bruteforce(q, k, v, g, beta, 0.6, h0, lib=lib)
    return max(_maxabs(a[0], b[0]), _maxabs(a[1], b[1]))


def pin_contraction(lib=None, seed=7):
    """For beta in [0,1], |k| = 1, alpha <= 1 the transition has spectral norm <= 1,
    so |S_t|_F <= |S_{t-1}|_F + beta |k| |v|.  Returns the largest excess (0 if held)."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=40, decay=0.05)
    S = h0
    worst = 0.0
    for t in range(q.shape[1]):
        sl = slice(t, t + 1)
        _, S_new = oracle.kda_fwd(q[:, sl], k[:, sl], v[:, sl], g[:, sl], beta[:, sl], 1.0, S, lib=lib)
        bound = (np.linalg.norm(S, axis=(-2, -1))
                 + beta[:, t] * np.linalg.norm(v[:, t], axis=-1))
        worst = max(worst, float(np.max(np.linalg.norm(S_new, axis=(-2, -1)) - bound)))
        S = S_new
    return max(worst, 0.0)


def pin_linearity_and_columns(lib=None, seed=8):
    """The map (v, h0) -> (out, hT) is linear for fixed q, k, g, beta, and the dv
    columns evolve independently (permuting v/h0 columns permutes out/hT)."""
    rng = np.random.default_rng(seed)
    q, k, v1, g, beta, h01 = rand_case(rng, T=21)
    v2 = rng.standard_normal(v1.shape)
    h02 = rng.standard_normal(h01.shape)
    a, b = 0.7, -1.9
    o1, s1 = oracle.kda_fwd(q, k, v1, g, beta, 0.5, h01, lib=lib)
    o2, s2 = oracle.kda_fwd(q, k, v2, g, beta, 0.5, h02, lib=lib)
    o3, s3 = oracle.kda_fwd(q, k, a * v1 + b * v2, g, beta, 0.5, a * h01 + b * h02, lib=lib)
    worst = max(_maxabs(o3, a * o1 + b * o2), _maxabs(s3, a * s1 + b * s2))
    perm = rng.permutation(v1.shape[-1])
    o4, s4 = oracle.kda_fwd(q, k, v1[..., perm], g, beta, 0.5, h01[..., perm], lib=lib)
    return max(worst, _maxabs(o4, o1[..., perm]), _maxabs(s4, s1[..., perm]))


def pin_continuation(lib=None, seed=9):
    """run(T1) then run(T2) from its final state equals run(T1 + T2)."""
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, h0 = rand_case(rng, T=31)
    full_o, full_s = oracle.kda_fwd(q, k, v, g, beta, 0.9, h0, lib=lib)
    a, b = slice(0, 12), slice(12, 31)
    o1, s1 = oracle.kda_fwd(q[:, a], k[:, a], v[:, a], g[:, a], beta[:, a], 0.9, h0, lib=lib)
    o2, s2 = oracle.kda_fwd(q[:, b], k[:, b], v[:, b], g[:, b], beta[:, b], 0.9, s1, lib=lib)
    return max(_maxabs(np.concatenate([o1, o2], axis=1), full_o), _maxabs(s2, full_s))


PIN_TOL = {
    pin_worked_examples: 1e-14,
    pin_beta_zero_closed_form: 1e-13,
    pin_gated_linear_attention: 1e-12,
    pin_linear_attention: 1e-12,
    pin_write_then_read: 1e-13,
    pin_write_read_identity: 1e-13,
    pin_bruteforce: 1e-12,
    pin_contraction: 1e-12,
    pin_linearity_and_columns: 1e-12,
    pin_continuation: 0.0,
}
