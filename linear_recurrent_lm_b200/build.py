"""Build libwkv7.so (the sm_100a CUDA library behind include/wkv7.h) in-tree with nvcc, and its
bounds-checked twin libwkv7_debug.so (same ABI, compiled with WKV7_DEBUG)."""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ = os.path.join(ROOT, "_build", "obj")
LIB = os.path.join(HERE, "libwkv7.so")
LIB_DEBUG = os.path.join(HERE, "libwkv7_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", f"-I{INCLUDE}", "-Xptxas", "-warn-spills"]


def _nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found; the WKV-7 library needs the CUDA toolkit to build")
    return exe


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


VARIANTS = {
    # name: (library, object folder, extra nvcc flags)
    "release": (LIB, OBJ, []),
    # every kernel index checked against its buffer; a failed check sets a status bit (WKV7_ERR_BOUNDS)
    "debug": (LIB_DEBUG, OBJ + "_debug", ["-DWKV7_DEBUG"]),
}


def build(force: bool = False, verbose: bool = False, variant: str = "release") -> str:
    """Compile every csrc/*.cu for sm_100a and link the variant's library; return its path."""
    lib, objdir, extra = VARIANTS[variant]
    nvcc = _nvcc()
    os.makedirs(objdir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(INCLUDE, "wkv7.h")]
    objs = []
    jobs = []
    for src in sources:
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, [src] + headers):
            jobs.append([nvcc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj])
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        for cmd, res in zip(jobs, ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs)):
            if verbose or res.returncode != 0:
                sys.stderr.write(res.stdout + res.stderr)
            if res.returncode != 0:
                raise RuntimeError(f"nvcc failed: {' '.join(cmd)}")
    if force or jobs or _stale(lib, objs):
        tmp = lib + ".tmp"
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError(f"linking {os.path.basename(lib)} failed")
        os.replace(tmp, lib)
    return lib


def build_all(force: bool = False, verbose: bool = False):
    """Both variants: libwkv7.so (release) and libwkv7_debug.so (bounds-checked)."""
    return [build(force, verbose, v) for v in VARIANTS]


if __name__ == "__main__":
    if "--debug" in sys.argv:
        print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, variant="debug"))
    elif "--release" in sys.argv:
        print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    else:
        print("\n".join(build_all(force="--force" in sys.argv, verbose="-v" in sys.argv)))
