"""Build the seeded-input generator libraries (host C and sm_100a device)."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _newer(out: str, *srcs: str) -> bool:
    return os.path.exists(out) and all(os.path.getmtime(out) >= os.path.getmtime(s) for s in srcs)


def build_host(force: bool = False) -> str:
    src = os.path.join(HERE, "gen_host.c")
    out = os.path.join(HERE, "libmoe_gen_host.so")
    if force or not _newer(out, src):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                               "-pthread", src, "-o", out])
    return out


def build_device(force: bool = False) -> str:
    src = os.path.join(HERE, "gen_device.cu")
    out = os.path.join(HERE, "libmoe_gen_device.so")
    if force or not _newer(out, src):
        subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
                               "-fmad=false", "-shared", "-Xcompiler", "-fPIC", src, "-o", out])
    return out


def build(force: bool = False) -> None:
    build_host(force)
    build_device(force)


if __name__ == "__main__":
    build(force=True)
