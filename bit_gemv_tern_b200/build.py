"""Builds bit_gemv_tern_b200/libterngemv.so in-tree with nvcc for sm_100a.

Each .cu file compiles to an object in _build/ (in parallel), then they link into one shared
library exporting the C ABI of include/tern.h.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build", "terngemv")
OUT = os.path.join(HERE, "libterngemv.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps() -> list[str]:
    hdr = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    return hdr + [os.path.join(ROOT, "include", "tern.h"), os.path.abspath(__file__)]


def _compile(src: str, obj: str, extra: list[str]) -> None:
    nvcc = os.environ.get("NVCC", "nvcc")
    subprocess.run([nvcc, *FLAGS, *ARCH, *extra, "-c", src, "-o", obj], check=True)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    srcs = sources()
    newest = max(os.path.getmtime(p) for p in srcs + _deps())
    if not force and not verbose_ptxas and os.path.exists(OUT) and os.path.getmtime(OUT) >= newest:
        return OUT
    os.makedirs(BUILD, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    objs = [os.path.join(BUILD, os.path.basename(s)[:-3] + ".o") for s in srcs]
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        list(ex.map(lambda so: _compile(so[0], so[1], extra), zip(srcs, objs)))
    nvcc = os.environ.get("NVCC", "nvcc")
    subprocess.run([nvcc, "-shared", *ARCH, "-o", OUT + ".tmp", *objs, "-lcudart"], check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
