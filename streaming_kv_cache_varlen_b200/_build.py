"""Build the CUDA library in-tree with nvcc for sm_100a.

The shared library statically links the CUDA runtime and exports only the
``cmp_*`` entry points declared in include/cmp.h, so it can be loaded next to
any other CUDA runtime (for example PyTorch's) without symbol clashes.
"""

from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libcmp_b200.so")
# measurement build: the same sources with the decode kernel's phase stamps
# (-DCMP_PHASE_STAMPS), for bench.py --only decode-phases
PHASES_OBJDIR = os.path.join(PKG, "_build", "phases")
PHASES_LIB = os.path.join(PKG, "libcmp_b200_phases.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
                 "-Xcompiler", "-fPIC,-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    nvcc = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return nvcc


def _newest_header() -> float:
    hs = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return max([os.path.getmtime(h) for h in hs] + [0.0])


def _compile(src: str, obj: str, extra: list, verbose: bool) -> None:
    cmd = [_nvcc(), *CFLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)


def build(verbose: bool = False, force: bool = False, ptxas_info: bool = False,
          phases: bool = False) -> str:
    """Compile every csrc/*.cu and link libcmp_b200.so (with phases=True the
    phase-stamp measurement build, libcmp_b200_phases.so). Returns the library path."""
    objdir, lib = (PHASES_OBJDIR, PHASES_LIB) if phases else (OBJDIR, LIB)
    os.makedirs(objdir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr = _newest_header()
    extra = (["-Xptxas", "-v"] if ptxas_info else []) + (["-DCMP_PHASE_STAMPS"] if phases else [])
    jobs = []
    for s in srcs:
        o = os.path.join(objdir, os.path.basename(s)[:-3] + ".o")
        if force or ptxas_info or not os.path.exists(o) or \
                os.path.getmtime(o) < max(os.path.getmtime(s), hdr):
            jobs.append((s, o))
    if jobs:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
            list(ex.map(lambda so: _compile(so[0], so[1], extra, verbose or ptxas_info), jobs))
    objs = [os.path.join(objdir, os.path.basename(s)[:-3] + ".o") for s in srcs]
    if jobs or force or not os.path.exists(lib):
        cmd = [_nvcc(), *ARCH, "-shared", "-o", lib, *objs, "-cudart", "static",
               "-Xlinker", "--exclude-libs,ALL", "-Xlinker", "-Bsymbolic", "-lrt", "-ldl",
               "-lpthread"]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


if __name__ == "__main__":
    import sys
    print(build(verbose="-v" in sys.argv, force="-f" in sys.argv,
                ptxas_info="--ptxas" in sys.argv, phases="--phases" in sys.argv))
