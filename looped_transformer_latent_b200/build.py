"""Build step: compile the CUDA sources into the in-tree shared library.

    python -m looped_transformer_latent_b200.build [--force]

produces ``looped_transformer_latent_b200/liblla.so`` for sm_100a (B200) with
nvcc.  The library is rebuilt when any source or header is newer than it.
"""

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblla.so")

SOURCES = ["abi.cu", "writer.cu", "decode_simt.cu", "decode_tc.cu", "decode_fp8.cu", "maps.cu", "gemm_tc.cu",
           "recon_tc.cu", "noalloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build liblla.so")


def _inputs():
    srcs = [os.path.join(CSRC, s) for s in SOURCES if os.path.exists(os.path.join(CSRC, s))]
    deps = list(srcs)
    for d in (CSRC, INCLUDE):
        for f in os.listdir(d):
            if f.endswith((".cuh", ".h")):
                deps.append(os.path.join(d, f))
    return srcs, deps


def needs_build():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    _, deps = _inputs()
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, verbose=False):
    """Compile liblla.so if it is missing or stale; return its path."""
    if not force and not needs_build():
        return LIB
    srcs, _ = _inputs()
    tmp = LIB + ".tmp"
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I", CSRC,
           *srcs, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
