"""Build of libdcpcombine.so, in-tree, for sm_100a.

    python -m decode_context_attention_dcp_b200._build        # build if stale
    python -m decode_context_attention_dcp_b200._build --force

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically, so it does not depend on which libcudart the host process loaded.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import glob
import hashlib
import os
import shutil
import subprocess
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
CSRC = os.path.join(PKG, "csrc")
LIBRARY = os.path.join(PKG, "libdcpcombine.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2"]
LINK_FLAGS = ["-shared", "--cudart", "static"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the DCP combine library needs the CUDA toolkit to build")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def inputs() -> list[str]:
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + sorted(glob.glob(os.path.join(INCLUDE, "*.h")))


def source_digest() -> str:
    """SHA-256 of every input's bytes and of the compiler flags: a library built from other
    sources (or a pushed library newer than its sources) is rebuilt, whatever the mtimes say."""
    h = hashlib.sha256()
    h.update(" ".join(ARCH + COMPILE_FLAGS + LINK_FLAGS).encode())
    for p in inputs():
        h.update(b"\0" + os.path.relpath(p, ROOT).encode() + b"\0")
        with open(p, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _digest_file(lib: str) -> str:
    return lib + ".sha256"


def stale(lib: str = LIBRARY) -> bool:
    """True unless ``lib`` exists and was built from exactly the current sources and flags."""
    if not os.path.exists(lib) or not os.path.exists(_digest_file(lib)):
        return True
    with open(_digest_file(lib)) as fh:
        return fh.read().strip() != source_digest()


def _run(cmd: list[str]) -> None:
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu under csrc/ (in parallel, one object each) and link them into one
    shared library (atomic replace)."""
    if not force and not stale():
        return LIBRARY
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=PKG)
    os.close(fd)
    objdir = tempfile.mkdtemp(prefix="dcp_build_")
    srcs = sources()
    objs = [os.path.join(objdir, os.path.basename(src) + ".o") for src in srcs]
    compiles = [[nvcc(), *ARCH, *COMPILE_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
                for src, obj in zip(srcs, objs)]
    link = [nvcc(), *ARCH, *LINK_FLAGS, "-o", tmp, *objs]
    try:
        with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
            for f in [ex.submit(_run, c) for c in compiles]:
                f.result()
        _run(link)
        if verbose:
            for c in compiles + [link]:
                print(" ".join(c))
        digest = source_digest()
        os.replace(tmp, LIBRARY)
        with open(_digest_file(LIBRARY) + ".tmp", "w") as fh:
            fh.write(digest + "\n")
        os.replace(_digest_file(LIBRARY) + ".tmp", _digest_file(LIBRARY))
    finally:
        if os.path.exists(tmp):
            os.unlink(tmp)
        shutil.rmtree(objdir, ignore_errors=True)
    return LIBRARY

if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=True))
