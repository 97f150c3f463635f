"""Build the CUDA library ``libhyena.so`` in-tree for sm_100a with nvcc, and its
debug twin ``libhyena_checked.so`` (the same sources with HYENA_CHECK_BOUNDS:
index checks that record a device error bit instead of accessing out of
range)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libhyena.so")
LIB_CHECKED = os.path.join(PKG, "libhyena_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def _object_stale(obj: str, dep: str, src: str, flags_file: str, flags: str) -> bool:
    """Whether an object must be rebuilt: missing, built with other flags, or older than its
    source or any file its dependency list (nvcc -MD) names."""
    if not (os.path.exists(obj) and os.path.exists(dep) and os.path.exists(flags_file)):
        return True
    with open(flags_file) as f:
        if f.read() != flags:
            return True
    t = os.path.getmtime(obj)
    with open(dep) as f:
        text = f.read().replace("\\\n", " ")
    deps = text.split(":", 1)[1].split() if ":" in text else [src]
    return any(not os.path.exists(d) or os.path.getmtime(d) > t for d in deps + [src])


def build(force: bool = False, verbose: bool = False, extra_flags=(), checked: bool = False) -> str:
    """Compile csrc/*.cu (in parallel, one object each; only the objects whose source or
    included headers changed) and link one shared library. Skipped when the library is
    newer than every source. checked=True builds the HYENA_CHECK_BOUNDS library."""
    lib = LIB_CHECKED if checked else LIB
    if checked:
        extra_flags = [*extra_flags, "-DHYENA_CHECK_BOUNDS"]
    if not force and not needs_build(lib):
        return lib
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    objdir = os.path.join(PKG, "_build_checked" if checked else "_build")
    os.makedirs(objdir, exist_ok=True)
    procs = []
    objs = []
    flags = " ".join([*NVCC_FLAGS, *extra_flags])
    for src in _sources():
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        dep, flags_file = obj[:-2] + ".d", obj[:-2] + ".flags"
        objs.append(obj)
        if not force and not _object_stale(obj, dep, src, flags_file, flags):
            continue
        if os.path.exists(flags_file):
            os.remove(flags_file)            # written back only once the object is built
        cmd = [nvcc, *NVCC_FLAGS, *extra_flags, "-I", INCLUDE, "-I", CSRC, "-MD", "-MF", dep, "-c", "-o", obj, src]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        procs.append((src, flags_file, subprocess.Popen(cmd)))
    failed = []
    for src, flags_file, p in procs:
        if p.wait() != 0:
            failed.append(src)
        else:
            with open(flags_file, "w") as f:
                f.write(flags)
    if failed:
        raise RuntimeError("nvcc failed on: " + ", ".join(failed))
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs, "-lcudart"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


def source_hash() -> str:
    """Hash of every source the library is built from (ties profiles to a kernel version)."""
    import hashlib
    hsh = hashlib.sha256()
    for p in _deps():
        hsh.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            hsh.update(f.read())
    return hsh.hexdigest()[:16]


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [], checked="--checked" in sys.argv))
