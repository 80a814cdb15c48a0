"""Build libpa_b200.so in-tree for sm_100a with nvcc.

Each translation unit under csrc/ is compiled in parallel into _build/, then
linked into paged_kv_cache_338_b200/libpa_b200.so with the CUDA runtime linked
statically and its symbols kept private (so the library's runtime never
resolves against another copy loaded in the same process).

``--nvtx`` compiles in an NVTX range around every C-ABI call that enqueues
work (for an Nsight Systems timeline; off by default).  The defines of the
last build are kept in _build/defines.txt; a build with other defines
recompiles everything.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libpa_b200.so")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                     "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(f for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def _headers_mtime() -> float:
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    hs.append(os.path.join(INCLUDE, "pa.h"))
    return max(os.path.getmtime(h) for h in hs)


def _compile(src: str, verbose_ptxas: bool, defines: list) -> str:
    obj = os.path.join(BUILD, src + ".o")
    path = os.path.join(CSRC, src)
    if (os.path.exists(obj) and os.path.getmtime(obj) >= os.path.getmtime(path)
            and os.path.getmtime(obj) >= _headers_mtime() and not verbose_ptxas):
        return obj
    cmd = [nvcc()] + NVCC_FLAGS + [f"-D{d}" for d in defines] + ["-c", path, "-o", obj + ".tmp"]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    os.replace(obj + ".tmp", obj)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False, jobs: int | None = None,
          nvtx: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sources()
    defines = ["PA_WITH_NVTX"] if nvtx else []
    stamp = os.path.join(BUILD, "defines.txt")
    old = open(stamp).read() if os.path.exists(stamp) else ""
    if old != " ".join(defines):
        force = True
    if force:
        for s in srcs:
            o = os.path.join(BUILD, s + ".o")
            if os.path.exists(o):
                os.remove(o)
    jobs = jobs or min(len(srcs), os.cpu_count() or 4)
    with cf.ThreadPoolExecutor(jobs) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas, defines), srcs))
    with open(stamp, "w") as f:
        f.write(" ".join(defines))
    if os.path.exists(LIB) and all(os.path.getmtime(LIB) >= os.path.getmtime(o) for o in objs):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs + [
        "-Xlinker", "--exclude-libs,ALL", "-Xlinker", "-Bsymbolic", "-lpthread", "-ldl", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv,
                nvtx="--nvtx" in sys.argv))
