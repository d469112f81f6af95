"""Build the layer's CUDA library (sm_100a) in-tree with nvcc.

``python -m fine_grained_shared_b200.csrc.build`` (or ``build()``) compiles
``moe_api.cu`` and the kernel headers it includes into
``fine_grained_shared_b200/libfgs_moe.so``.  nvcc cross-compiles for sm_100a
without a GPU present.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libfgs_moe.so")
SOURCES = ["moe_api.cu", "route_noalloc.cu", "fp8_quant.cu"]
HEADERS = ["sm100.cuh", "router_topk.cuh", "permute.cuh", "gateup_gemm.cuh", "down_gemm.cuh", "decode_ffn.cuh",
           "fp8_util.cuh", "fp8_gemm.cuh", "decode_ffn8.cuh", "ep_plan.h", "ep.cuh"]


def nvcc_path() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def flags(extra=()):
    return ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
            "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
            "-I", os.path.join(ROOT, "include"), *extra]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = [os.path.join(HERE, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "fgs_moe.h"),
                                                                    os.path.abspath(__file__)]
    return all(os.path.getmtime(p) <= t for p in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    if not force and not ptxas_info and up_to_date():
        return LIB
    cmd = [nvcc_path(), *flags(["-Xptxas", "-v"] if ptxas_info else []),
           *[os.path.join(HERE, s) for s in SOURCES], "-o", LIB + ".tmp"]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libfgs_moe.so")
    if verbose or ptxas_info:
        sys.stderr.write(res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv)
