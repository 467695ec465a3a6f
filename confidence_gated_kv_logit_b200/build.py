"""Build libconfkv.so (the CUDA library behind include/confkv.h) in-tree.

nvcc compiles every translation unit under csrc/ for sm_100a (in parallel)
and links a shared library next to this file. The runtime is linked
statically, so the library needs only the driver at run time.
"""
from __future__ import annotations

import glob
import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libconfkv.so")
STAMP = LIB + ".sha256"

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-Xcudafe", "--diag_suppress=177",
]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def source_digest() -> str:
    """Hash of every input of the build (sources, headers, flags)."""
    deps = sorted(sources() + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + glob.glob(os.path.join(HERE, "csrc", "*.h")))
    deps.append(os.path.join(ROOT, "include", "confkv.h"))
    h = hashlib.sha256(" ".join(NVCC_FLAGS).encode())
    for d in deps:
        h.update(os.path.relpath(d, ROOT).encode())
        with open(d, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def needs_build() -> bool:
    if not os.path.exists(LIB) or not os.path.exists(STAMP):
        return True
    with open(STAMP) as f:
        return f.read().strip() != source_digest()


def build_checked(verbose: bool = False) -> str:
    """Build libconfkv_checked.so: the same library with every data-dependent
    index checked on the device (failures are recorded and skipped)."""
    out = os.path.join(HERE, "libconfkv_checked.so")
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    cmd = [nvcc, *NVCC_FLAGS, "-DCONFKV_CHECKED", "-shared", "-I", os.path.join(ROOT, "include"), "-o", out, *sources()]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed to build libconfkv_checked.so")
    return out


def build(verbose: bool = False, ptxas_info: bool = False, force: bool = False) -> str:
    """Compile every translation unit to an object (in parallel), then link
    the shared library."""
    if not force and not needs_build():
        return LIB
    import tempfile
    from concurrent.futures import ThreadPoolExecutor
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    with tempfile.TemporaryDirectory(prefix="confkv_build_") as tmp:
        def compile_one(src):
            obj = os.path.join(tmp, os.path.basename(src) + ".o")
            cmd = [nvcc, *extra, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            return obj, subprocess.run(cmd, capture_output=True, text=True)
        with ThreadPoolExecutor(max_workers=max(1, min(len(sources()), os.cpu_count() or 1))) as ex:
            results = list(ex.map(compile_one, sources()))
        for _, res in results:
            if res.returncode != 0:
                sys.stderr.write(res.stdout + res.stderr)
                raise RuntimeError("nvcc failed to build libconfkv.so")
            if ptxas_info or verbose:
                sys.stdout.write(res.stdout + res.stderr)
        link = [nvcc, *NVCC_FLAGS, "-shared", "-o", LIB + ".tmp", *[o for o, _ in results]]
        if verbose:
            print(" ".join(link), flush=True)
        res = subprocess.run(link, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError("nvcc failed to link libconfkv.so")
    os.replace(LIB + ".tmp", LIB)
    with open(STAMP, "w") as f:
        f.write(source_digest())
    return LIB


if __name__ == "__main__":
    build(verbose=True, ptxas_info="-v" in sys.argv, force=True)
