"""Build libssmscan.so (sm_100a) in-tree from csrc/*.cu with nvcc."""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libssmscan.so")
OBJDIR = os.path.join(HERE, "_build")
# the same sources with the device index checks compiled in (-DSSM_DEBUG)
DEBUG_LIB = os.path.join(HERE, "libssmscan_debug.so")
DEBUG_OBJDIR = os.path.join(HERE, "_build_debug")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE,
         "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, out: str | None = None,
          defines: tuple = ()) -> str:
    """Compile csrc/*.cu into `out` (default: the in-tree libssmscan.so)."""
    lib = out or LIB
    objdir = OBJDIR if out is None else out + ".objs"
    if out is None and not force and not defines and up_to_date():
        return LIB
    if out == DEBUG_LIB:
        objdir = DEBUG_OBJDIR
    os.makedirs(objdir, exist_ok=True)
    cc = nvcc()
    srcs = _sources()
    objs = [os.path.join(objdir, os.path.basename(s)[:-3] + ".o") for s in srcs]

    def comp(pair):
        s, o = pair
        cmd = [cc, *ARCH, *FLAGS, *[f"-D{d}" for d in defines], "-c", s, "-o", o]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {s}:\n{r.stderr}")
        return r.stderr

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        logs = list(ex.map(comp, zip(srcs, objs)))
    if verbose:
        print("\n".join(logs))
    tmp = lib + f".tmp{os.getpid()}"
    # cudart linked statically: the library does not depend on which CUDA
    # runtime (if any) the host process loaded.
    subprocess.run([cc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs], check=True)
    os.replace(tmp, lib)
    return lib


def build_debug(force: bool = False) -> str:
    """Compile the debug library (device index checks, -DSSM_DEBUG) in-tree;
    select it at run time with SSM_LIBRARY=<its path>."""
    if not force and up_to_date(DEBUG_LIB):
        return DEBUG_LIB
    return build(force=True, out=DEBUG_LIB, defines=("SSM_DEBUG",))


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", action="store_true")
    ap.add_argument("--out", default=None, help="write the library here instead of in-tree")
    ap.add_argument("-D", action="append", default=[], help="preprocessor define (repeatable)")
    ap.add_argument("--debug", action="store_true", help="build the debug library (index checks)")
    a = ap.parse_args()
    if a.debug:
        print(build_debug(force=a.force))
    else:
        print(build(force=a.force, verbose=a.v, out=a.out, defines=tuple(a.D)))
