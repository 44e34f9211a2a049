"""Builds the generator's host library (gcc) and device library (nvcc, sm_100a).

The host build disables floating-point contraction and the device build disables
fused multiply-add, so both evaluate the synth_core.h series with the same IEEE
roundings and produce identical bits.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
BUILD = os.path.join(HERE, "_build")
HOST_LIB = os.path.join(BUILD, "libsynth_host.so")
DEV_LIB = os.path.join(BUILD, "libsynth_dev.so")


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build_host(force=False):
    srcs = [os.path.join(HERE, "synth_host.c"), os.path.join(HERE, "synth_core.h")]
    if force or _stale(HOST_LIB, srcs):
        os.makedirs(BUILD, exist_ok=True)
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-Wall", "-o", HOST_LIB, srcs[0], "-lpthread", "-lm"])
    return HOST_LIB


def build_dev(force=False):
    srcs = [os.path.join(HERE, "synth_dev.cu"), os.path.join(HERE, "synth_core.h")]
    if force or _stale(DEV_LIB, srcs):
        os.makedirs(BUILD, exist_ok=True)
        subprocess.check_call(["nvcc", "-O2", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                               "-fmad=false", "-cudart", "static",
                               "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                               "-o", DEV_LIB, srcs[0]])
    return DEV_LIB


def build(force=False):
    build_host(force)
    build_dev(force)


if __name__ == "__main__":
    build(force=True)
