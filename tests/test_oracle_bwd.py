"""Pins of the oracle's backward pass (kda_oracle_bwd), CPU only.

The backward is the plain definition: the gradient of
L = sum(dout * out) + sum(dhT * hT) through the forward recurrence.  It is
pinned to things other than itself:

* central finite differences of the forward oracle, entry by entry, for every
  input (q, k, v, g, the erase and write weights, h0) on tiny problems;
* two exact identities from the method's linearity: out is linear in q and
  hT does not depend on q, so <dq, q> = sum(dout * out); and (out, hT) are
  jointly linear in (v, h0), so <dv, v> + <dh0, h0> = L;
* planted mistakes in a copy of the C source, each of which must break one of
  the above.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")


def problem(seed, B=1, T=5, H=2, dk=3, dv=4, beta_one=False):
    rng = np.random.default_rng(seed)
    x = dict(q=rng.standard_normal((B, T, H, dk)), k=rng.standard_normal((B, T, H, dk)) * 0.6,
             v=rng.standard_normal((B, T, H, dv)),
             g=-0.5 * np.log1p(np.exp(rng.standard_normal((B, T, H, dk)))),
             erase=1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H)))),
             write=1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H)))),
             h0=rng.standard_normal((B, H, dk, dv)) * 0.5)
    if beta_one:
        x["erase"] = np.ones((B, T, H))
        x["write"] = np.ones((B, T, H))
        x["k"] /= np.linalg.norm(x["k"], axis=-1, keepdims=True)
    dout = rng.standard_normal((B, T, H, dv))
    dhT = rng.standard_normal((B, H, dk, dv))
    return x, dout, dhT


def loss(x, dout, dhT, scale, lib=None):
    out, hT = oracle.kda_fwd(x["q"], x["k"], x["v"], x["g"], None, scale, x["h0"], erase=x["erase"],
                             write=x["write"], threads=1, lib=lib)
    return float(np.sum(dout * out) + np.sum(dhT * hT))


def grads(x, dout, dhT, scale, lib=None):
    return oracle.kda_bwd(x["q"], x["k"], x["v"], x["g"], None, scale, x["h0"], dout, dhT, erase=x["erase"],
                          write=x["write"], threads=1, lib=lib)


NAMES = {"q": "dq", "k": "dk", "v": "dv", "g": "dg", "erase": "derase", "write": "dwrite", "h0": "dh0"}


def fd_error(seed, lib=None, **kw):
    """Largest |analytic - central difference| / (1 + |analytic|) over every entry."""
    scale = 0.7
    x, dout, dhT = problem(seed, **kw)
    gr = grads(x, dout, dhT, scale, lib=lib)
    eps = 1e-6
    worst = 0.0
    for name, gname in NAMES.items():
        a = x[name]
        for idx in np.ndindex(a.shape):
            old = a[idx]
            a[idx] = old + eps
            lp = loss(x, dout, dhT, scale)
            a[idx] = old - eps
            lm = loss(x, dout, dhT, scale)
            a[idx] = old
            fd = (lp - lm) / (2 * eps)
            an = gr[gname][idx]
            worst = max(worst, abs(an - fd) / (1.0 + abs(an)))
    return worst


def identity_error(seed, lib=None, **kw):
    """The two linearity identities, relative to the loss."""
    scale = 0.7
    x, dout, dhT = problem(seed, **kw)
    gr = grads(x, dout, dhT, scale, lib=lib)
    out, _ = oracle.kda_fwd(x["q"], x["k"], x["v"], x["g"], None, scale, x["h0"], erase=x["erase"],
                            write=x["write"], threads=1)
    L = loss(x, dout, dhT, scale)
    e1 = abs(np.sum(gr["dq"] * x["q"]) - np.sum(dout * out)) / (1.0 + abs(np.sum(dout * out)))
    e2 = abs(np.sum(gr["dv"] * x["v"]) + np.sum(gr["dh0"] * x["h0"]) - L) / (1.0 + abs(L))
    return max(e1, e2)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_backward_matches_finite_differences(seed):
    assert fd_error(seed) < 1e-6


def test_backward_matches_finite_differences_beta_one_unit_keys():
    """beta = 1 with unit keys: the erase makes (I - k k^T) singular along k."""
    assert fd_error(3, beta_one=True) < 1e-6


def test_backward_linearity_identities():
    for seed in range(4):
        assert identity_error(seed, B=2, T=17, H=2, dk=5, dv=3) < 1e-10


def test_backward_without_dout_or_dhT():
    """Either cotangent may be absent: the gradients are those of the other part."""
    x, dout, dhT = problem(7)
    full = grads(x, dout, dhT, 0.7)
    a = oracle.kda_bwd(x["q"], x["k"], x["v"], x["g"], None, 0.7, x["h0"], dout, None, erase=x["erase"],
                       write=x["write"], threads=1)
    b = oracle.kda_bwd(x["q"], x["k"], x["v"], x["g"], None, 0.7, x["h0"], None, dhT, erase=x["erase"],
                       write=x["write"], threads=1)
    for n in ("dq", "dk", "dv", "dg", "derase", "dwrite", "dh0"):
        np.testing.assert_allclose(a[n] + b[n], full[n], rtol=1e-12, atol=1e-12)
    assert np.all(b["dq"] == 0.0)


BWD_MUTANTS = {
    "readout_before_write": ("acc += S1[r * dv + c] * dout[row * dv + c];",
                             "acc += S0[r * dv + c] * dout[row * dv + c];"),
    "adjoint_not_decayed": ("dS[r * dv + c] *= a;", ""),
    "projection_term_dropped": ("dkt[r] += acc;", ""),
    "erase_grad_sign": ("det -= du[c] * p[c];", "det += du[c] * p[c];"),
    "gate_grad_without_alpha": ("dgt[r] = a * acc;", "dgt[r] = acc;"),
    "write_grad_uses_erase": ("dvt[c] = wt * du[c];", "dvt[c] = et * du[c];"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    start = src.index("int kda_oracle_bwd(")
    end = src.index("int kda_oracle_max_threads(")
    body = src[start:end]
    assert body.count(old) == 1, f"{name}: pattern not found once in the backward"
    mutated = src[:start] + body.replace(old, new) + src[end:]
    c_path, so_path = tmp_path / f"{name}.c", tmp_path / f"lib{name}.so"
    c_path.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    "-o", str(so_path), str(c_path), "-lm"], check=True)
    return oracle.load_library(str(so_path))


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_backward_mutant_is_caught(tmp_path, name):
    lib = _build_mutant(tmp_path, name, *BWD_MUTANTS[name])
    assert fd_error(0, lib=lib) > 1e-4 or identity_error(0, lib=lib) > 1e-6
