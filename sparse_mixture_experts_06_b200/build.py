"""Builds libmoe.so in-tree with nvcc for sm_100a (B200).

    python sparse_mixture_experts_06_b200/build.py [--force] [-v]

(run by path: importing the package would load the library being rebuilt)

Each csrc/*.cu is compiled to an object under _build/ (rebuilt when the
source, a header or the flags change) and linked into a shared library that
exports only the moe_* C ABI of include/moe.h.  The CUDA runtime is linked
statically; the driver API is reached through cudaGetDriverEntryPoint, so no
libcuda link is needed and the build runs on a machine without a GPU.
"""

from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build", "moe")
LIB = os.path.join(PKG, "libmoe.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3", "-Xptxas", "-v",
                 "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found (set NVCC or install the CUDA toolkit)")


def _digest(paths, extra) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as fh:
            h.update(fh.read())
    h.update(" ".join(extra).encode())
    return h.hexdigest()[:16]


def compile_objects(sources, headers, flags, build_dir, verbose=False, force=False):
    os.makedirs(build_dir, exist_ok=True)
    objs = []
    for src in sources:
        tag = _digest([src] + headers, flags)
        obj = os.path.join(build_dir, os.path.basename(src) + "." + tag + ".o")
        if force or not os.path.exists(obj):
            cmd = [nvcc()] + flags + ["-c", src, "-o", obj]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, " ".join(cmd), r.stderr))
            with open(obj + ".log", "w") as fh:
                fh.write(r.stderr)
            if verbose:
                sys.stderr.write(r.stderr)
        objs.append(obj)
    return objs


def link_shared(objs, out, export_prefix):
    vs = os.path.join(os.path.dirname(objs[0]), export_prefix + "exports.map")
    with open(vs, "w") as fh:
        fh.write("{ global: %s*; local: *; };\n" % export_prefix)
    tmp = out + ".tmp"
    cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs + \
        ["-Xlinker", "--version-script=" + vs, "-lpthread", "-ldl", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s\n%s" % (" ".join(cmd), r.stderr))
    os.replace(tmp, out)


def build(verbose: bool = False, force: bool = False) -> str:
    sources = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))
    headers = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")) + \
        [os.path.join(ROOT, "include", "moe.h")]
    objs = compile_objects(sources, headers, CFLAGS, BUILD, verbose, force)
    link_shared(objs, LIB, "moe_")
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force="--force" in sys.argv))
