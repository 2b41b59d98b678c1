"""Build the CUDA library in-tree: csrc/*.cu -> libstq.so (sm_100a only).

``python -m quantized_linear_attention_stq_b200.build`` or ``build()`` from Python. The library
is rebuilt when a source or the public header is newer than the shared object.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
HEADER = os.path.join(ROOT, "include", "stq.h")
LIB = os.path.join(PKG, "libstq.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-Xptxas", "-warn-spills"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libstq.so")


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [HEADER]
    return os.path.getmtime(LIB) < max(os.path.getmtime(f) for f in deps)


def _compile(src: str, obj: str, ptxas_info: bool):
    cmd = [_nvcc(), *ARCH, *FLAGS, "-c", "-o", obj, src]
    if ptxas_info:
        cmd += ["-Xptxas", "-v"]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    return cmd, proc


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    """Compile every source to an object (in parallel, under the package's _build folder), then
    link libstq.so. Objects whose source and headers are older than them are reused."""
    if not (force or stale()):
        return LIB
    from concurrent.futures import ThreadPoolExecutor

    objdir = os.path.join(ROOT, "_build", "stq")
    os.makedirs(objdir, exist_ok=True)
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + [HEADER]
    newest_header = max(os.path.getmtime(f) for f in headers)
    jobs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        fresh = os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(src), newest_header)
        jobs.append((src, obj, force or not fresh))
    todo = [j for j in jobs if j[2]]
    with ThreadPoolExecutor(max_workers=max(1, min(len(todo), os.cpu_count() or 1))) as ex:
        results = list(ex.map(lambda j: _compile(j[0], j[1], ptxas_info), todo))
    for (src, _, _), (cmd, proc) in zip(todo, results):
        if verbose:
            print(" ".join(cmd), flush=True)
        if proc.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src} ({proc.returncode}):\n{proc.stdout}\n{proc.stderr}")
        if verbose or ptxas_info:
            sys.stdout.write(proc.stdout + proc.stderr)
    tmp = LIB + f".tmp{os.getpid()}"
    link = [_nvcc(), *ARCH, "-shared", "-o", tmp, *[j[1] for j in jobs]]
    proc = subprocess.run(link, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError(f"nvcc link failed ({proc.returncode}):\n{proc.stdout}\n{proc.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas-info" in sys.argv)
