"""Build liblf_hsa.so in place: every kernel compiled for sm_100a with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

_HERE = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_HERE)
SOURCES = ["lf_api.cu", "lf_pool.cu", "lf_select.cu", "lf_ivf.cu", "lf_quant.cu", "lf_attn.cu"]
HEADERS = ["lf_device.cuh", "lf_internal.h", "lf_score.cuh"]
LIB = os.path.join(_HERE, "liblf_hsa.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(_HERE, "csrc", f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(_ROOT, "include", "lf_hsa.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    if not force and not ptxas_info and not _stale():
        return LIB
    srcs = [os.path.join(_HERE, "csrc", f) for f in SOURCES]
    tmp = LIB + ".tmp"
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", os.path.join(_ROOT, "include"), "-shared",
           "-cudart", "static", "-o", tmp, *srcs, "-ldl", "-lrt", "-lpthread"]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True, ptxas_info="-v" in sys.argv))
