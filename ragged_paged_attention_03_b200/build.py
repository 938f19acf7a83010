"""Build librpa_b200.so in-tree: every .cu under csrc/ compiled for sm_100a by
nvcc (in parallel, rebuilt only when a source or header changed), then linked
into one shared library with the CUDA runtime linked statically."""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "librpa_b200.so")
# Timing-only variant for bench.py --ablate-write: the fused cache stores
# compiled out (RPA_ABLATE_CACHE_WRITE); never loaded by the product binding
# unless RPA_ABLATE_CACHE_WRITE=1 is set in the environment.
NOWRITE_OBJ = os.path.join(HERE, "_build_nowrite")
NOWRITE_LIB = os.path.join(HERE, "librpa_b200_nowrite.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, verbose_ptxas=False, obj_dir=OBJ, defines=()):
    obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, *[f"-D{d}" for d in defines], "-c", src, "-o", obj]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stderr}")
    return obj, r.stderr


def build(force: bool = False, verbose_ptxas: bool = False, jobs: int = 0, ablate_write: bool = False) -> str:
    obj_dir, lib = (NOWRITE_OBJ, NOWRITE_LIB) if ablate_write else (OBJ, LIB)
    defines = ("RPA_ABLATE_CACHE_WRITE",) if ablate_write else ()
    os.makedirs(obj_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdrs = _headers()
    todo = [s for s in sources
            if force or verbose_ptxas or _stale(os.path.join(obj_dir, os.path.basename(s) + ".o"), [s, *hdrs])]
    logs = {}
    if todo:
        with cf.ThreadPoolExecutor(max_workers=jobs or min(8, os.cpu_count() or 1)) as ex:
            for src, (obj, err) in zip(todo, ex.map(lambda s: _compile(s, verbose_ptxas, obj_dir, defines), todo)):
                logs[src] = err
    objs = [os.path.join(obj_dir, os.path.basename(s) + ".o") for s in sources]
    if todo or _stale(lib, objs):
        tmp = lib + f".{os.getpid()}.tmp"
        subprocess.check_call([NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs])
        os.replace(tmp, lib)
    if verbose_ptxas:
        for src, err in logs.items():
            print(f"== {os.path.basename(src)}\n{err}")
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv,
                ablate_write="--ablate-write" in sys.argv))
