"""Builds libwukong.so (the C ABI of include/wukong.h) for sm_100a, in-tree.

nvcc -gencode arch=compute_100a,code=sm_100a -O3 -lineinfo, static CUDA runtime,
so the library loads (and exports its symbols) on a machine without a GPU and
uses the caller's CUDA context when there is one.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "_lib", "libwukong.so")
SOURCES = ["wk_api.cu"]
HEADERS = ["common.cuh", "gemm_tc.cuh", "gemm_tc2.cuh", "lcb_tc.cuh", "fm_tc.cuh", "front_tc.cuh", "res_ln.cuh", "res_ln_ring.cuh", "simt.cuh", "convert.cuh", "moe.cuh", "head.cuh", "whale.cuh", "backward.cuh", "bw_tc.cuh"]


def _stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "wukong.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def nvcc_flags():
    return ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-cudart", "static",
            "-I" + INCLUDE, "-I" + CSRC, "--expt-relaxed-constexpr", "-Xptxas", "-v"]


def build(force=False, verbose=False):
    if not force and not _stale():
        return LIB
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    cmd = ["nvcc", "-shared"] + nvcc_flags() + ["-o", LIB] + [os.path.join(CSRC, s) for s in SOURCES]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    with open(os.path.join(os.path.dirname(LIB), "ptxas.log"), "w") as f:
        f.write(r.stdout + r.stderr)
    if verbose:
        print(r.stdout + r.stderr)
    return LIB


if __name__ == "__main__":
    build(force=True)
    print(LIB)
