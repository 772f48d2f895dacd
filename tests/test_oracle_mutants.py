"""Planted mistakes in the oracle must each break at least one pin.

Each case copies ``oracle/kda_oracle.c``, applies one plausible mistake to the
token-by-token recurrence (a dropped term, a wrong sign, a wrong operand, the
wrong order of decay / erase / read), builds it with gcc into a temporary
directory and runs every pin against that build.  The shipped oracle is not
modified.  CPU only.
"""
import os
import subprocess

import pytest

import oracle
from oracle_pins import PIN_TOL

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

DECAY = """                double a = exp(gt[r]);
                for (long c = 0; c < dv; ++c) S[r * dv + c] *= a;"""

MUTANTS = {
    "erase_dropped": ("u[c] = wt * vt[c] - et * p[c];", "u[c] = wt * vt[c];"),
    "erase_sign": ("u[c] = wt * vt[c] - et * p[c];", "u[c] = wt * vt[c] + et * p[c];"),
    "erase_uses_write_weight": ("u[c] = wt * vt[c] - et * p[c];", "u[c] = wt * vt[c] - wt * p[c];"),
    "write_uses_erase_weight": ("u[c] = wt * vt[c] - et * p[c];", "u[c] = et * vt[c] - et * p[c];"),
    "decay_sign": ("double a = exp(gt[r]);", "double a = exp(-gt[r]);"),
    "decay_on_value_columns": (DECAY, "                for (long c = 0; c < dv; ++c) S[r * dv + c] *= exp(gt[c % dk]);"),
    "projection_uses_query": ("p[c] += kt[r] * S[r * dv + c];", "p[c] += qt[r] * S[r * dv + c];"),
    "read_before_write": ("ot[c] += qt[r] * S[r * dv + c];", "ot[c] += qt[r] * (S[r * dv + c] - kt[r] * u[c]);"),
    "read_before_decay": ("ot[c] += qt[r] * S[r * dv + c];",
                          "ot[c] += qt[r] * ((S[r * dv + c] - kt[r] * u[c]) / exp(gt[r]) + kt[r] * u[c]);"),
    "scale_dropped": ("for (long c = 0; c < dv; ++c) ot[c] *= scale;", ""),
    "h0_ignored": ("if (h0) memcpy(S, h0 + bh * dk * dv, sizeof(double) * dk * dv);",
                   "if (0) memcpy(S, h0 + bh * dk * dv, sizeof(double) * dk * dv);"),
    "update_transposed_index": ("S[r * dv + c] += kt[r] * u[c];", "S[r * dv + c] += kt[c % dk] * u[r % dv];"),
    "decay_after_write": (DECAY, ""),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"{name}: pattern not found"
    body_start = src.index("int kda_oracle_fwd(")
    body_end = src.index("int kda_oracle_bruteforce(")
    body = src[body_start:body_end]
    assert old in body, f"{name}: pattern not in the recurrence"
    body = body.replace(old, new, 1)
    if name == "decay_after_write":
        # move the per-channel decay after the write (and before the read)
        body = body.replace("            /* 5. readout after the write",
                            "            for (long r = 0; r < dk; ++r) {\n" + DECAY + "\n            }\n"
                            "            /* 5. readout after the write", 1)
    mutated = src[:body_start] + body + src[body_end:]
    c_path = tmp_path / f"{name}.c"
    so_path = tmp_path / f"lib{name}.so"
    c_path.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    "-o", str(so_path), str(c_path), "-lm"], check=True)
    return oracle.load_library(str(so_path))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    lib = _build_mutant(tmp_path, name, old, new)
    caught = []
    for pin, tol in PIN_TOL.items():
        try:
            err = pin(lib=lib)
        except Exception as exc:  # a mutant that breaks the oracle outright also counts
            caught.append(f"{pin.__name__}: {exc!r}")
            continue
        if not err <= tol:
            caught.append(f"{pin.__name__}: {err:.2e}")
    assert caught, f"mutant {name} passed every pin"
