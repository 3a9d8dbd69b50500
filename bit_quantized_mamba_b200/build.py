"""Build libdfssm.so (the sm_100a CUDA library behind include/dfssm.h) in-tree with nvcc."""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libdfssm.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr", "-I", INCLUDE]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + [
        os.path.join(os.path.dirname(HERE), "include", "dfssm.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in _deps())


def _compile(src: str, verbose: bool, obj_dir: str = OBJ, extra=()) -> str:
    obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and r.stderr:
        print(r.stderr, file=sys.stderr)
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJ, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose), sources()))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


CPU_SRC = os.path.join(HERE, "cpu", "dfssm_cpu.cpp")
CPU_LIB = os.path.join(HERE, "libdfssm_cpu.so")


def build_cpu(force: bool = False) -> str:
    """libdfssm_cpu.so: the host-CPU (AVX-512 VNNI) engine (include/dfssm_cpu.h).  The VNNI code sits in
    functions compiled for that target and is entered only after a run-time CPU check; the rest is
    built for the baseline x86-64 target with no contraction of products and sums."""
    deps = [CPU_SRC, os.path.join(INCLUDE, "dfssm_cpu.h"), os.path.join(INCLUDE, "dfssm.h")]
    if not force and os.path.exists(CPU_LIB) and all(os.path.getmtime(d) <= os.path.getmtime(CPU_LIB) for d in deps):
        return CPU_LIB
    tmp = CPU_LIB + f".tmp{os.getpid()}"
    cmd = ["g++", "-O3", "-std=c++17", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
           "-I", INCLUDE, CPU_SRC, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"g++ failed for {CPU_SRC}:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, CPU_LIB)
    return CPU_LIB


def build_trace() -> str:
    """libdfssm_trace.so: the same library with the fused decode kernel's phase stamps compiled in
    (-DDFSSM_TRACE_DECODE); used by trace_decode.py only."""
    out = os.path.join(HERE, "libdfssm_trace.so")
    obj_dir = os.path.join(HERE, "_build_trace")
    os.makedirs(obj_dir, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        objs = list(ex.map(lambda s: _compile(s, False, obj_dir, ("-DDFSSM_TRACE_DECODE",)), sources()))
    r = subprocess.run([NVCC, *ARCH, "-shared", "-o", out, *objs], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    print(build_cpu(force="--force" in sys.argv))
