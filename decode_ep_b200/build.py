"""Builds libentropack.so in-tree: the sm_100a decode kernel, the host encoder and the C ABI.

    python -m decode_ep_b200.build          # or: python decode_ep_b200/build.py

Device code is compiled for sm_100a only. The encoder is compiled with -ffp-contract=off, because
its estimates and quantisation decisions must be plain IEEE double arithmetic.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libentropack.so")
SOURCES = ["decode.cu", "host_encoder.cpp", "capi.cpp", "plan.cpp", "tans_host.cpp"]
# Compiled on their own with --fmad=false: the CUDA encoder must round every double operation alone.
NOFMA_SOURCES = ["gpu_encoder.cu"]
HEADERS = ["epk_format.h", "capi_internal.h", "encoder_common.h", "lattice_code.h", "tans_format.h", "tans_decode.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the EntroPack CUDA library cannot be built")


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + NOFMA_SOURCES + HEADERS] + [os.path.join(ROOT, "include", "entropack.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    common = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC,-ffp-contract=off,-O3",
              "-I", os.path.join(ROOT, "include"), "-I", CSRC]
    with tempfile.TemporaryDirectory() as tmp:
        objs = []
        for f in NOFMA_SOURCES:
            obj = os.path.join(tmp, f + ".o")
            cmd = [nvcc(), *common, "--fmad=false", "-c", os.path.join(CSRC, f), "-o", obj]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            subprocess.run(cmd, check=True)
            objs.append(obj)
        cmd = [nvcc(), *common, "-shared", *[os.path.join(CSRC, f) for f in SOURCES], *objs,
               "-o", LIB + ".tmp", "-lpthread"]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
