"""Build the sm_100a shared library in-tree: scaled_dot_product_bwd_b200/libsdpa_b200.so.

    python -m scaled_dot_product_bwd_b200.build [--verbose]

nvcc cross-compiles for sm_100a without a GPU.  The CUDA runtime is linked
statically so the library needs only the driver at run time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libsdpa_b200.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)
SOURCES = ["sdpa_api.cu"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    out = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh", ".h"))]
    out.append(os.path.join(INCLUDE, "sdpa.h"))
    return out


STAMP_PATH = LIB_PATH + ".stamp"


def _source_hash(flags) -> str:
    import hashlib
    h = hashlib.sha256(" ".join(flags).encode())
    for d in sorted(_deps()):
        if os.path.isfile(d):
            h.update(os.path.relpath(d, ROOT).encode())
            with open(d, "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()


def up_to_date(flags=()) -> bool:
    """The library exists and was built from exactly these sources and flags."""
    if not (os.path.exists(LIB_PATH) and os.path.exists(STAMP_PATH)):
        return False
    with open(STAMP_PATH) as fh:
        return fh.read().strip() == _source_hash(flags)


FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-gencode", "arch=compute_100a,code=sm_100a",
         "-Xcompiler", "-fPIC", "-shared", "-cudart", "static"]


def source_hash() -> str:
    """Hash of the kernel sources and build flags the library is built from."""
    return _source_hash(FLAGS)


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and up_to_date(FLAGS):
        return LIB_PATH
    cmd = [nvcc_path()] + FLAGS + [
        "-I", INCLUDE, "-I", CSRC,
        "-o", LIB_PATH + ".tmp",
    ] + [os.path.join(CSRC, s) for s in SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(LIB_PATH + ".tmp", LIB_PATH)
    with open(STAMP_PATH, "w") as fh:
        fh.write(_source_hash(FLAGS) + "\n")
    return LIB_PATH


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    print(LIB_PATH)
