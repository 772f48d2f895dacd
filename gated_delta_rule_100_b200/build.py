"""Build libkda.so (sm_100a) in-tree with nvcc, and libkda_debug.so, the same
sources compiled with KDA_DEBUG (device-side index checks that report
KDA_ERR_BOUNDS instead of trapping; for tests).

    python -m gated_delta_rule_100_b200.build [--force]

The shared libraries are written next to this file so they travel with the
source tree; nothing is installed into site-packages.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB_PATH = os.path.join(HERE, "libkda.so")
DEBUG_LIB_PATH = os.path.join(HERE, "libkda_debug.so")
SOURCES = ["kda_api.cu", "decode.cu", "prep_fwd.cu", "exact_prep.cu", "chain_fwd.cu", "varlen_setup.cu", "parts_fixup.cu", "bwd.cu", "host_fwd.cu"]
HEADERS = ["kda_device.cuh", "chunk_common.cuh", "chunk_params.cuh", "bwd_params.cuh"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _inputs():
    return ([os.path.join(CSRC, s) for s in SOURCES + HEADERS]
            + [os.path.join(INCLUDE, "kda.h")])


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def _build_one(lib_path: str, defines, subdir: str, verbose: bool) -> None:
    build_dir = os.path.join(HERE, "_build", subdir)
    os.makedirs(build_dir, exist_ok=True)
    objs, procs = [], []
    for src in SOURCES:
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        cmd = [_nvcc(), *NVCC_FLAGS, *defines, "-I", INCLUDE, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append(subprocess.Popen(cmd))
        objs.append(obj)
    for p in procs:
        if p.wait() != 0:
            raise RuntimeError(f"nvcc failed building {os.path.basename(lib_path)}")
    tmp = lib_path + f".tmp{os.getpid()}"
    cmd = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib_path)


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Build libkda.so (and, unless debug is False, libkda_debug.so) when stale."""
    if force or not up_to_date(LIB_PATH):
        _build_one(LIB_PATH, [], "release", verbose)
    if debug and (force or not up_to_date(DEBUG_LIB_PATH)):
        _build_one(DEBUG_LIB_PATH, ["-DKDA_DEBUG"], "debug", verbose)
    return LIB_PATH


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=True))


if __name__ == "__main__":
    sys.exit(main())
