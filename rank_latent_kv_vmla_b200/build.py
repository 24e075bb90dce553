"""Build libvmla.so in-tree with nvcc for sm_100a.

    python -m rank_latent_kv_vmla_b200.build [--force] [--jobs N] [--checked]

Objects go to ``_build/`` at the repository root; the shared library is written next to this file.
Whether an object or the library is current is decided by content, not by modification times: each
object records a SHA-256 of its source, every header, this script and the compiler flags, and the
library records the hashes of the objects it was linked from (``<lib>.sha256``).  A build whose
recorded hash differs, or is missing, is redone, so objects or libraries carried over from another
checkout are never used as they are.
``--checked`` builds ``libvmla_checked.so`` (objects in ``_build_checked/``) with VMLA_CHECKED=1: every
computed global store of the tensor-core kernels is tested against its buffer's extent (a store outside
is skipped and reported in the device status word).  Select it with VMLA_LIBRARY=<path> at import.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libvmla.so")
BUILD_CHECKED = os.path.join(ROOT, "_build_checked")
LIB_CHECKED = os.path.join(PKG, "libvmla_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden", "--expt-relaxed-constexpr",
              "-I", INCLUDE, "-I", CSRC] + ARCH


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libvmla")
    return path


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _flags_key(flags) -> list:
    """The compiler flags without this checkout's paths (a checkout elsewhere hashes the same), plus the
    compiler's version."""
    rel = [os.path.relpath(f, ROOT) if os.path.isabs(f) else f for f in flags]
    return rel + [_nvcc_version()]


_NVCC_VERSION = []


def _nvcc_version() -> str:
    if not _NVCC_VERSION:
        r = subprocess.run([nvcc(), "--version"], capture_output=True, text=True)
        _NVCC_VERSION.append(r.stdout.strip().splitlines()[-1] if r.returncode == 0 and r.stdout.strip() else "")
    return _NVCC_VERSION[0]


def _digest(paths, extra) -> str:
    h = hashlib.sha256()
    for p in paths:
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    h.update(repr(list(extra)).encode())
    return h.hexdigest()


def _recorded(target: str) -> str:
    try:
        with open(target + ".sha256") as f:
            return f.read().strip()
    except OSError:
        return ""


def _record(target: str, digest: str) -> None:
    with open(target + ".sha256", "w") as f:
        f.write(digest + "\n")


def _compile(src: str, obj: str, extra):
    cmd = [nvcc(), "-c", src, "-o", obj] + NVCC_FLAGS + list(extra)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    return r.stderr


def build(force: bool = False, jobs: int = 0, extra=(), verbose: bool = False, checked: bool = False) -> str:
    build_dir, lib = (BUILD_CHECKED, LIB_CHECKED) if checked else (BUILD, LIB)
    extra = list(extra) + (["-DVMLA_CHECKED=1"] if checked else [])
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = _headers()
    objs, todo, digests = [], [], []
    common = sorted(headers) + [os.path.abspath(__file__)]
    for src in sources:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        digest = _digest([src] + common, _flags_key(NVCC_FLAGS + list(extra)))
        objs.append(obj)
        digests.append(digest)
        if force or not os.path.exists(obj) or _recorded(obj) != digest:
            todo.append((src, obj, digest))
    if todo:
        n = jobs or min(len(todo), os.cpu_count() or 1)
        with cf.ThreadPoolExecutor(max_workers=n) as ex:
            for (src, obj, digest), log in zip(todo, ex.map(lambda t: _compile(t[0], t[1], extra), todo)):
                _record(obj, digest)
                if verbose and log:
                    print(f"--- {os.path.basename(src)}\n{log}", file=sys.stderr)
    lib_digest = hashlib.sha256("".join(digests).encode()).hexdigest()
    if force or todo or not os.path.exists(lib) or _recorded(lib) != lib_digest:
        tmp = lib + ".tmp"
        cmd = [nvcc(), "-shared", "-o", tmp] + objs + ARCH
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
        _record(lib, lib_digest)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--jobs", type=int, default=0)
    ap.add_argument("--ptxas-verbose", action="store_true", help="print register/smem use per kernel")
    ap.add_argument("--checked", action="store_true", help="build libvmla_checked.so (bounds-checked stores)")
    a = ap.parse_args()
    extra = ["-Xptxas", "-v"] if a.ptxas_verbose else []
    print(build(force=a.force or a.ptxas_verbose, jobs=a.jobs, extra=extra, verbose=a.ptxas_verbose,
                checked=a.checked))


if __name__ == "__main__":
    main()
