"""Build libssta.so in-tree with nvcc for sm_100a.

    python block_sparse_video_ssta_b200/build.py [--verbose]   (does not import the package)

Each .cu under csrc/ compiles to an object in parallel, then one shared
library is linked next to this file (the CUDA runtime is linked statically, so
the library does not depend on which libcudart the host process loaded).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT = os.path.join(HERE, "libssta.so")
STAMP = OUT + ".sha256"   # hash of the sources the library was built from
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _source_hash(extra_flags=()) -> str:
    """sha256 over every source and header the library is built from, and the flags."""
    h = hashlib.sha256()
    deps = sources() + sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh")))
    deps.append(os.path.join(INCLUDE, "ssta.h"))
    for p in deps:
        h.update(os.path.relpath(p, ROOT).encode() + b"\0")
        with open(p, "rb") as f:
            h.update(f.read())
    h.update(" ".join(ARCH + FLAGS[:-4] + list(extra_flags)).encode())
    return h.hexdigest()


def _needs_rebuild() -> bool:
    """Rebuild unless the library exists and its stamp holds the current sources' hash
    (file times are not trusted: a copied tree can carry a library newer than its sources)."""
    if not (os.path.exists(OUT) and os.path.exists(STAMP)):
        return True
    with open(STAMP) as f:
        return f.read().strip() != _source_hash()


def build(verbose: bool = False, force: bool = False, ptxas_info: bool = False) -> str:
    if not force and not _needs_rebuild():
        return OUT
    os.makedirs(BUILD_DIR, exist_ok=True)
    cc = nvcc()
    extra = ["-Xptxas", "-v"] if ptxas_info else []

    def compile_one(src):
        obj = os.path.join(BUILD_DIR, os.path.basename(src)[:-3] + ".o")
        cmd = [cc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        return src, obj, r

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, sources()))
    failed = False
    for src, _, r in results:
        if verbose or r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
        if r.returncode != 0:
            sys.stderr.write(f"nvcc failed on {src}\n")
            failed = True
    if failed:
        raise RuntimeError("CUDA build failed")
    tmp = OUT + ".tmp"
    link = [cc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *[o for _, o, _ in results]]
    r = subprocess.run(link, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link failed")
    os.replace(tmp, OUT)
    with open(STAMP, "w") as f:
        f.write(_source_hash() + "\n")
    return OUT


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    a = ap.parse_args()
    print(build(verbose=a.verbose or a.ptxas_info, force=a.force, ptxas_info=a.ptxas_info))


if __name__ == "__main__":
    main()
