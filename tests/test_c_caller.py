"""The C ABI from a plain C99 program: tests/c_abi_caller.c includes only
include/wtconv.h and links only libwtconv.so (no torch, no Python).  It is
compiled with -Werror here and its host-side results (workspace and folded
sizes, launch counts, argument errors) must equal the same calls made
through the Python binding.  Nothing in it launches a kernel."""
import ctypes
import os
import shutil
import subprocess

import pytest

import depthwise_convolution_wtconv_b200 as wt
from depthwise_convolution_wtconv_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "depthwise_convolution_wtconv_b200")


@pytest.fixture(scope="module")
def c_results(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    wt.load()
    exe = str(tmp_path_factory.mktemp("c") / "c_abi_caller")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I" + os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_caller.c"), "-L" + PKG, "-lwtconv",
                    "-Wl,-rpath," + PKG, "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    return dict(line.split(" ", 1) for line in out.strip().splitlines())


def test_c_caller_sizes_and_launches_match_binding(c_results):
    lib = wt.load()
    d = _lib.WTConvDesc(2, 3, 16, 16, 5, 2, 0)
    for op in range(4):
        assert int(c_results[f"ws_{op}"]) == lib.wtconv_workspace_size(ctypes.byref(d), op) > 16
    ragged = _lib.WTConvDesc(2, 3, 16, 10, 5, 2, 1)
    assert int(c_results["ws_ragged_2"]) == lib.wtconv_workspace_size(ctypes.byref(ragged), 2)
    assert int(c_results["ws_even_k"]) == 0
    assert int(c_results["folded"]) == lib.wtconv_folded_size(ctypes.byref(d)) > 0
    for op in range(6):
        assert int(c_results[f"launches_{op}"]) == lib.wtconv_kernel_launches(ctypes.byref(d), op) > 0


def test_c_caller_gets_host_side_errors(c_results):
    assert int(c_results["fwd_null_x"]) == 1            # WTCONV_ERR_ARG
    assert int(c_results["fwd_even_k"]) == 1            # WTCONV_ERR_ARG
    assert int(c_results["fwd_small_ws"]) == 4          # WTCONV_ERR_WORKSPACE
    assert int(c_results["bwd_data_misaligned"]) == 3   # WTCONV_ERR_ALIGN
    assert int(c_results["noalloc_ragged"]) == 2        # WTCONV_ERR_SHAPE
    assert int(c_results["noalloc_huge_c"]) == 7        # WTCONV_ERR_SCRATCH_LIMIT
    assert c_results["status_string_ok"] == "set"
    # the array size the header promises is the one the library was built with
    assert int(c_results["scratch_bytes"]) == int(c_results["scratch_macro"]) == _lib.noalloc_scratch_bytes()
    assert c_results["status_string_limit"] == "set"


def test_same_caller_as_cxx_links_through_extern_c(c_results, tmp_path):
    """C++ callers get the unmangled symbols through the header's extern "C"
    block: the caller built as C++17 prints the same results."""
    if shutil.which("g++") is None:
        pytest.skip("no C++ compiler")
    exe = str(tmp_path / "cxx_abi_caller")
    subprocess.run(["g++", "-x", "c++", "-std=c++17", "-Wall", "-Wextra", "-Werror",
                    "-I" + os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_caller.c"),
                    "-L" + PKG, "-lwtconv", "-Wl,-rpath," + PKG, "-o", exe], check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    assert dict(line.split(" ", 1) for line in out.strip().splitlines()) == c_results
