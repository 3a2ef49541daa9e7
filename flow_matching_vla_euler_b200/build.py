"""Builds the sm_100a shared library libvla_b200.so in-tree with nvcc.

    python -m flow_matching_vla_euler_b200.build [--verbose-ptxas]

Each .cu under csrc/ is compiled to an object (in parallel), then linked with the static
CUDA runtime into a C-ABI shared library next to this file. The SHA-256 of the sources,
headers and flags it was built from is written beside it (libvla_b200.so.sha256); a
later build() reuses the library only when that hash matches. The driver API entry point
used for TMA descriptors is fetched at run time, so the library links no libcuda.
"""
from __future__ import annotations

import concurrent.futures as cf
import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libvla_b200.so")
LIB_HASH = LIB + ".sha256"   # source hash the library was built from
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _compile(src: str, verbose_ptxas: bool) -> str:
    obj = os.path.join(BUILD, os.path.basename(src) + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, "-c", src, "-o", obj]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    return obj


def source_hash(srcs, headers) -> str:
    """SHA-256 over every source and header (by name and content), the compiler flags and
    this script: the library is rebuilt whenever any of them differs from what it was
    built from, whatever the file times say."""
    h = hashlib.sha256()
    for f in sorted(srcs + headers + [os.path.abspath(__file__)]):
        h.update(os.path.basename(f).encode() + b"\0")
        with open(f, "rb") as fh:
            h.update(fh.read())
    h.update(" ".join(ARCH + FLAGS[:-1]).encode())
    return h.hexdigest()


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sources()
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    headers.append(os.path.join(INCLUDE, "vla.h"))
    want = source_hash(srcs, headers)
    if not force and os.path.exists(LIB) and os.path.exists(LIB_HASH):
        with open(LIB_HASH) as f:
            if f.read().strip() == want:
                return LIB
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas), srcs))
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    with open(LIB_HASH, "w") as f:
        f.write(want + "\n")
    return LIB


if __name__ == "__main__":
    print(build(verbose_ptxas="--verbose-ptxas" in sys.argv, force=True))
