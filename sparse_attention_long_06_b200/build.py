"""Build the sm_100a library libnsa_b200.so in-tree with nvcc.

Usage: python -m sparse_attention_long_06_b200.build [--force]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libnsa_b200.so")
SOURCES = ["nsa_api.cu", "nsa_noalloc.cu", "k_prep.cu", "k_cmp.cu", "k_win.cu", "k_slc.cu",
           "k_decode.cu", "k_bsel.cu", "k_compress.cu", "k_dsa.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the sm_100a library cannot be built")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES]
    files += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")]
    files.append(os.path.join(os.path.dirname(PKG), "include", "nsa.h"))
    return files


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not is_stale():
        return LIB
    nvcc = _nvcc()
    with tempfile.TemporaryDirectory(prefix="nsa_build_") as tmp:
        objs = []
        procs = []
        for src in SOURCES:
            obj = os.path.join(tmp, src.replace(".cu", ".o"))
            cmd = [nvcc, *ARCH, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
            if verbose:
                cmd += ["-Xptxas", "-v"]
            procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
            objs.append(obj)
        failed = False
        for src, p in procs:
            out, _ = p.communicate()
            if p.returncode != 0 or verbose:
                sys.stderr.write(out.decode(errors="replace"))
            failed |= p.returncode != 0
        if failed:
            raise RuntimeError("nvcc failed while building libnsa_b200.so")
        tmp_lib = os.path.join(tmp, "libnsa_b200.so")
        subprocess.check_call([nvcc, *ARCH, "-shared", "-o", tmp_lib, *objs])
        shutil.copyfile(tmp_lib, LIB + ".tmp")
        os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
