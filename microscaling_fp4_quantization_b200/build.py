"""Build the native library lib/libfp4q.so (sm_100a) in-tree with nvcc.

    python -m microscaling_fp4_quantization_b200.build
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIB_DIR, "libfp4q.so")

# The C ABI and its dispatch, then one unit per kernel family (compiled in parallel).
SOURCES = ["fp4q.cu", "fp4q_inst_rq_mx.cu", "fp4q_inst_rq_nv.cu", "fp4q_inst_mbs.cu", "fp4q_inst_qe.cu",
           "fp4q_inst_mma.cu", "fp4q_inst_mma_qe.cu", "fp4q_inst_dequant.cu", "fp4q_inst_gemm.cu"]
DEPS = SOURCES + ["fp4q_kernels.cuh", "fp4q_device.cuh", "fp4q_mma.cuh", "fp4q_host.cuh", "fp4q_launch.cuh", "fp4q_gemm.cuh"]
OBJ_DIR = os.path.join(PKG, "lib", "obj")


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def flags():
    return ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++20",
            "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-O2", "-I", INCLUDE, "-I", CSRC]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(INCLUDE, "fp4q.h"), __file__]
    return all(os.path.getmtime(d) <= t for d in deps)


def _compile(src: str, obj: str, verbose: bool) -> str:
    cmd = [nvcc(), *flags(), "-c", "-o", obj, os.path.join(CSRC, src)]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src} ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    return r.stdout + r.stderr


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    objs = [os.path.join(OBJ_DIR, os.path.splitext(src)[0] + ".o") for src in SOURCES]
    jobs = max(1, min(len(SOURCES), os.cpu_count() or 1))
    with ThreadPoolExecutor(max_workers=jobs) as pool:
        logs = list(pool.map(lambda so: _compile(so[0], so[1], verbose), zip(SOURCES, objs)))
    if verbose:
        print("".join(logs))
    tmp = LIB + ".tmp"
    # every symbol must resolve inside the library: a launcher instantiated nowhere fails here
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xlinker", "--no-undefined",
           "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
