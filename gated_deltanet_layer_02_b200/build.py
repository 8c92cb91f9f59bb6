"""Build libgdn.so in-tree for sm_100a with nvcc (no JIT cache, nothing installed).

    python -m gated_deltanet_layer_02_b200.build [--force] [--bounds-check]

Each .cu under csrc/ is compiled to an object in csrc/_build/ (rebuilt when it or a header is
newer), then linked into gated_deltanet_layer_02_b200/libgdn.so with the CUDA runtime linked
statically.  ``--bounds-check`` builds the checked variant instead: every source compiled with
-DGDN_BOUNDS_CHECK into csrc/_build_checked/ and linked into libgdn_checked.so (index checks
in the kernels that record GDN_ERR_BOUNDS in the caller's status word and skip the access).
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(CSRC, "_build")
LIB = os.path.join(HERE, "libgdn.so")
BUILD_CHECKED = os.path.join(CSRC, "_build_checked")
LIB_CHECKED = os.path.join(HERE, "libgdn_checked.so")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, bounds_check: bool = False) -> str:
    nvcc = _nvcc()
    build_dir, lib_path = (BUILD_CHECKED, LIB_CHECKED) if bounds_check else (BUILD, LIB)
    flags = FLAGS + (["-DGDN_BOUNDS_CHECK"] if bounds_check else [])
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    headers = _headers()
    jobs = []
    for src in sources:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        if force or _stale(obj, [src] + headers):
            jobs.append((src, obj))

    def compile_one(job):
        src, obj = job
        cmd = [nvcc, *ARCH, *flags, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stderr}")
        return r.stderr

    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(8, len(jobs)))) as ex:
        for msg in ex.map(compile_one, jobs):
            if verbose and msg:
                sys.stderr.write(msg)
    objs = [os.path.join(build_dir, os.path.basename(s)[:-3] + ".o") for s in sources]
    if force or jobs or _stale(lib_path, objs):
        tmp = lib_path + f".{os.getpid()}.tmp"
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stderr}")
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                bounds_check="--bounds-check" in sys.argv))
