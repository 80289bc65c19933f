"""Build liblowbit.so (sm_100a) in-tree with nvcc.

The library is rebuilt when the SHA-1 of its sources and flags changes, so a
stale binary can never be loaded after the sources move on.  Usage:

    python -m decode_packed_bit_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import os
import re
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblowbit.so")
STAMP = os.path.join(PKG, ".liblowbit.sha1")
OBJDIR = os.path.join(ROOT, "_build", "lowbit")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
          "-I" + INCLUDE, "-I" + CSRC]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def digest() -> str:
    h = hashlib.sha1()
    for p in sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(INCLUDE, "lowbit.h")]:
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    h.update(" ".join(ARCH + CFLAGS).encode())
    return h.hexdigest()


def _strip_c_comments(text: str) -> str:
    """C/C++ source with comments removed and whitespace runs collapsed (a
    string literal holding a comment marker would be cut too; the sources
    have none that matter for code identity)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_digest(files=None) -> str:
    """SHA-1 of CUDA sources' code alone (comments and layout stripped) and
    the compile flags: the key under which measured counters of a kernel
    (profiles/traffic.json) stay valid.  `files`: the csrc file names a
    kernel is compiled from (default: all of them).  Editing documentation
    does not change it; editing the code of those files does."""
    h = hashlib.sha1()
    paths = sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")))
    if files is not None:
        paths = [os.path.join(CSRC, f) for f in files]
    for p in paths:
        h.update(os.path.basename(p).encode())
        with open(p, encoding="utf-8") as f:
            h.update(_strip_c_comments(f.read()).encode())
    # the flags without include paths, which depend on where the tree lives
    h.update(" ".join(ARCH + [f for f in CFLAGS if not f.startswith("-I")]).encode())
    return h.hexdigest()


def build(force: bool = False, verbose: bool = False, out: str | None = None, defines=()) -> str:
    """Compile every csrc/*.cu and link liblowbit.so.  `out` and `defines`
    (extra -D flags) build a variant elsewhere, e.g. for a tuning sweep; the
    default is the in-tree library."""
    lib = out or LIB
    stamp = STAMP if out is None else out + ".sha1"
    objdir = OBJDIR if out is None else out + ".objs"
    d = digest() + "".join(" -D" + x for x in defines)
    if not force and os.path.exists(lib) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == d:
                return lib
    os.makedirs(objdir, exist_ok=True)
    extra = (["-Xptxas", "-v"] if verbose else []) + ["-D" + x for x in defines]

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *CFLAGS, *extra, "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
        if verbose and r.stderr:
            sys.stderr.write(r.stderr)
        return obj

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, sources()))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    with open(stamp, "w") as f:
        f.write(d + "\n")
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/spill report")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
