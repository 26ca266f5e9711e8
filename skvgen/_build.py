"""Compile the seeded input generator: host C library and device CUDA library."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(HERE, "libskvgen_host.so")
DEV_SO = os.path.join(HERE, "libskvgen_dev.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _stale(out, srcs):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(os.path.join(HERE, s)) > t for s in srcs)


def build(force=False, device=True):
    if force or _stale(HOST_SO, ["host.c", "core.h"]):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-o", HOST_SO, os.path.join(HERE, "host.c"), "-lm"])
    if device and (force or _stale(DEV_SO, ["device.cu", "core.h"])):
        subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                               "-lineinfo", "-shared", "-Xcompiler", "-fPIC", "-o", DEV_SO,
                               os.path.join(HERE, "device.cu")])


if __name__ == "__main__":
    build(force=True)
