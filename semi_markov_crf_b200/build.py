"""Build the C-ABI library ``libsemicrf_b200.so`` in-tree with nvcc (sm_100a).

Usage:  python -m semi_markov_crf_b200.build [--force] [--verbose] [--bounds-check]

``--bounds-check`` builds the debug variant ``libsemicrf_b200_check.so``
(-DSEMICRF_BOUNDS_CHECK): index checks in the kernels record the first
failing site in the workspace status word instead of making the access.
The binding loads it when SEMICRF_LIBRARY=check.

Compiles every ``csrc/*.cu`` for ``-gencode arch=compute_100a,code=sm_100a``
(with -lineinfo) and links a shared library with the CUDA runtime linked
statically, so the library needs only the driver at run time.  Rebuilds when
any source or header is newer than the library.  The sha256 of the kernel
sources (``source_digest()``) is compiled in: ``semicrf_source_digest()``
returns it, so a caller can tell a library built from other sources.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsemicrf_b200.so")
LIB_CHECK = os.path.join(PKG, "libsemicrf_b200_check.so")
BUILD_DIR = os.path.join(PKG, "_build")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    "-I", INCLUDE, "-I", CSRC,
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or put CUDA's bin on PATH)")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def source_digest() -> str:
    """sha256 over the kernel sources (csrc/*.cu, *.cuh: name, NUL, bytes, in
    name order)."""
    import hashlib
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, bounds_check: bool = False) -> str:
    lib = LIB_CHECK if bounds_check else LIB
    if not force and not _stale(lib):
        return lib
    nvcc = _nvcc()
    bdir = BUILD_DIR + ("_check" if bounds_check else "")
    os.makedirs(bdir, exist_ok=True)
    extra = ["-DSEMICRF_BOUNDS_CHECK"] if bounds_check else []
    extra.append(f'-DSEMICRF_SOURCE_DIGEST="{source_digest()}"')
    from concurrent.futures import ThreadPoolExecutor

    def compile_one(src):
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc, *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        res = subprocess.run(cmd, capture_output=True, text=True)
        if verbose or res.returncode:
            sys.stdout.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
            sys.stdout.flush()
        if res.returncode:
            raise subprocess.CalledProcessError(res.returncode, cmd)
        return obj

    with ThreadPoolExecutor(max(1, min(len(sources()), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(compile_one, sources()))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-cudart", "static",
           "-Xcompiler", "-fPIC", *objs, "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                bounds_check="--bounds-check" in sys.argv))
