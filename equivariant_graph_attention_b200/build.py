"""Compile libegat.so (sm_100a) in-tree with nvcc.

    python -m equivariant_graph_attention_b200.build [-v]

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` (rebuilt when
the source, a header or the flags change) and linked into
``equivariant_graph_attention_b200/libegat.so`` with the CUDA runtime linked
statically.  Only the ``egat_*`` symbols declared in ``include/egat.h`` are
exported.
"""
from __future__ import annotations

import glob
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libegat.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
                 "-Xcompiler", "-fPIC,-fvisibility=hidden,-O2", "-I", INCLUDE]


def _digest(paths, extra):
    h = hashlib.sha256()
    for p in sorted(paths):
        with open(p, "rb") as f:
            h.update(f.read())
    h.update(" ".join(extra).encode())
    return h.hexdigest()[:16]


def build(verbose: bool = False, ptxas_info: bool = False) -> str:
    """Build libegat.so if anything changed; return its path."""
    os.makedirs(BUILD, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                     + glob.glob(os.path.join(INCLUDE, "*.h")))
    flags = CFLAGS + (["-Xptxas", "-v"] if ptxas_info else [])
    objs = []
    for src in sources:
        tag = _digest([src] + headers, flags)
        obj = os.path.join(BUILD, f"{os.path.basename(src)}.{tag}.o")
        objs.append(obj)
        if os.path.exists(obj) and not ptxas_info:
            continue
        cmd = [NVCC] + flags + ["-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0 or verbose or ptxas_info:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}")
    link_tag = _digest(objs, ARCH)
    stamp = os.path.join(BUILD, "libegat.stamp")
    if os.path.exists(LIB) and os.path.exists(stamp) and open(stamp).read() == link_tag:
        return LIB
    tmp = LIB + ".tmp"
    cmd = [NVCC] + ARCH + ["-shared", "-o", tmp] + objs
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc link failed")
    os.replace(tmp, LIB)
    with open(stamp, "w") as f:
        f.write(link_tag)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, ptxas_info="--ptxas" in sys.argv))
