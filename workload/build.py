"""Builds the two twins of the synthetic-input generator.

``libwl_host.so`` (gcc, OpenMP, no fp contraction) and ``libwl_device.so``
(nvcc for sm_100a, no fused multiply-add) are compiled from ``wl_gen.h`` so
both produce the same bits for the same (seed, stream, element).
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(HERE, "libwl_host.so")
DEVICE_SO = os.path.join(HERE, "libwl_device.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(os.path.join(HERE, s)) > t for s in sources)


def build_host(force=False):
    if force or _stale(HOST_SO, ["wl_host.c", "wl_gen.h"]):
        tmp = HOST_SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-fPIC", "-shared", "-Wall",
                               os.path.join(HERE, "wl_host.c"), "-o", tmp, "-lm"])
        os.replace(tmp, HOST_SO)
    return HOST_SO


def build_device(force=False):
    if force or _stale(DEVICE_SO, ["wl_device.cu", "wl_gen.h"]):
        tmp = DEVICE_SO + ".tmp%d" % os.getpid()
        subprocess.check_call([NVCC, "-O3", "-gencode", "arch=compute_100a,code=sm_100a",
                               "--fmad=false", "-Xcompiler", "-fPIC", "-shared",
                               os.path.join(HERE, "wl_device.cu"), "-o", tmp])
        os.replace(tmp, DEVICE_SO)
    return DEVICE_SO


if __name__ == "__main__":
    print(build_host(force=True))
    print(build_device(force=True))
