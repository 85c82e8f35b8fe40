"""Builds libwtconv.so in-tree for sm_100a with nvcc.

    python -m depthwise_convolution_wtconv_b200.build
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = [os.path.join(PKG, "csrc", "wtconv_api.cu")]
DEPS = SRC + [os.path.join(PKG, "csrc", f) for f in os.listdir(os.path.join(PKG, "csrc"))] + [
    os.path.join(ROOT, "include", "wtconv.h")]
LIB = os.path.join(PKG, "libwtconv.so")


def nvcc_command(verbose=False):
    cmd = [
        "nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
        "-shared", "-Xcompiler", "-fPIC", "-I" + os.path.join(ROOT, "include"),
        "-I" + os.path.join(PKG, "csrc"), "-o", LIB,
    ] + SRC
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in DEPS if os.path.exists(p))


def build(force=False, verbose=False):
    if not force and up_to_date():
        return LIB
    subprocess.run(nvcc_command(verbose), check=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
