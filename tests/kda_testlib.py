"""Shared helpers for the parity tests: tolerances, error metrics, and running
the oracle on the same (bf16-rounded) inputs the CUDA path consumes."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Parity bar on every checked tensor (outputs and states), taken over the
# tensor as a whole: relative L2 error and largest absolute error.
REL_L2_TOL = 5e-3
MAX_ABS_TOL = 2e-2


def f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def rel_l2(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / den) if den > 0 else float(np.linalg.norm(x))


def max_abs(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref))) if x.size else 0.0


# Every comparison made by assert_close, in order: (what, rel-L2, max-abs, rel tol,
# max-abs tol).  conftest.py writes them to $KDA_PARITY_LOG (JSON) at the end of
# the session, so the precision margin of each check can be read off a run.
PARITY_LOG = []


def assert_close(x, ref, what, rel=REL_L2_TOL, mabs=MAX_ABS_TOL):
    r, m = rel_l2(x, ref), max_abs(x, ref)
    PARITY_LOG.append({"what": what, "rel_l2": r, "max_abs": m, "rel_tol": rel, "max_abs_tol": mabs})
    assert np.all(np.isfinite(np.asarray(x, np.float64))), f"{what}: non-finite values"
    assert r <= rel and m <= mabs, f"{what}: rel-L2 {r:.3e} (tol {rel:.1e}), max-abs {m:.3e} (tol {mabs:.1e})"
    return r, m


def oracle_prefill(d, scale, heads=None, tokens=None, batches=None, threads=None):
    """Oracle out/hT on (optionally) a slice of heads / leading tokens / batches of
    a prefill input dict (torch tensors, any device)."""
    sl_b = slice(None) if batches is None else batches
    sl_t = slice(None) if tokens is None else slice(0, tokens)
    sl_h = slice(None) if heads is None else heads

    def cut(t, has_t=True):
        if t is None:
            return None
        return f64(t[sl_b, sl_t, sl_h] if has_t else t[sl_b, sl_h])

    return oracle.kda_fwd(cut(d["q"]), cut(d["k"]), cut(d["v"]), cut(d["g"]), cut(d["beta"]),
                          scale, cut(d["h0"], has_t=False), threads=threads)
