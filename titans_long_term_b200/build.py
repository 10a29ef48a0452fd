"""Build libtitans_mem.so in-tree with nvcc for sm_100a.

    python -m titans_long_term_b200.build [--force] [--verbose-ptxas] [--debug]

``--debug`` builds libtitans_mem_debug.so instead, with -DTITANS_DEBUG: the tensor-core kernels then
check the runtime-dependent coordinates and offsets of their memory accesses and report a failed
check in the device status word (bit 8) instead of making the access. The binding loads it when the
environment variable TITANS_DEBUG is 1.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libtitans_mem.so")
BUILD_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libtitans_mem_debug.so")
SOURCES = ["api.cu", "chunk_cuda_cores.cu", "chunk_deep_cuda_cores.cu", "chunk_tc_mlp64.cu", "chunk_tc_phased.cu",
           "chunk_tc_deep.cu", "step_cluster.cu", "forward_noalloc.cu", "linear_scan.cu",
           "linear_backward.cu", "mlp_backward.cu", "mlp_backward_tc.cu"]
HEADERS = ["kernels.h", "ptx.cuh", "phased_common.cuh"]
NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         f"-I{os.path.join(ROOT, 'include')}", "--expt-relaxed-constexpr"]


def _stale(out: str, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False, debug: bool = False) -> str:
    build_dir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD, LIB)
    flags = FLAGS + (["-DTITANS_DEBUG"] if debug else [])
    os.makedirs(build_dir, exist_ok=True)
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "titans_mem.h")]
    jobs = []
    for s in SOURCES:
        src = os.path.join(CSRC, s)
        obj = os.path.join(build_dir, s.replace(".cu", ".o"))
        if force or verbose_ptxas or _stale(obj, [src] + hdrs):
            cmd = [NVCC, *ARCH, *flags, "-c", src, "-o", obj]
            if verbose_ptxas:
                cmd += ["-Xptxas", "-v"]
            jobs.append(cmd)
    objs = [os.path.join(build_dir, s.replace(".cu", ".o")) for s in SOURCES]

    def run(cmd):
        return subprocess.run(cmd, capture_output=True, text=True)

    with cf.ThreadPoolExecutor(max_workers=min(4, max(1, len(jobs)))) as ex:
        for cmd, res in zip(jobs, ex.map(run, jobs)):
            if res.returncode != 0:
                sys.stderr.write(res.stdout + res.stderr)
                raise RuntimeError(f"nvcc failed: {' '.join(cmd)}")
            if verbose_ptxas:
                sys.stderr.write(res.stderr)
    if force or jobs or _stale(lib, objs):
        cmd = [NVCC, *ARCH, "-shared", "-o", lib, *objs, "-lcuda"]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError("link failed")
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv,
                debug="--debug" in sys.argv))
