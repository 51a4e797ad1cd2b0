"""Host checks of the kernels' work-distribution arithmetic (csrc/tile_sched.h).

The stream-K ranges of the weight-streaming kernels, their launch plan (how
many split-K partial slots a column group needs), the split-K-in-a-cluster
plan that replaces stream-K where it fills the GPU, the CTA-pair kernel's
hybrid schedule (whole tiles, then split halves of a thin last wave), the
grouped raster of the
persistent tile kernels and the fp32 split-K ranges are plain integer
arithmetic shared by the device code and the launchers.  A wrong range here
drops or double-counts part of the k sum, or leaves tiles unwritten, on some
shapes only; these tests walk whole parameter grids on the CPU instead.
"""
import ctypes
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "tiled_dense_gemm_tma_b200", "csrc")


@pytest.fixture(scope="module")
def chk(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    out = str(tmp_path_factory.mktemp("sched") / "libsched_check.so")
    subprocess.run([gxx, "-O2", "-std=c++17", "-shared", "-fPIC", "-I", CSRC,
                    os.path.join(HERE, "sched_check.cpp"), "-o", out], check=True)
    lib = ctypes.CDLL(out)
    ll = ctypes.c_longlong
    for name, args in (("check_stream_k", [ctypes.c_int, ctypes.c_int]),
                       ("check_stream_k_large", []),
                       ("check_sk_plan", []),
                       ("check_tile_coords", [ctypes.c_int, ctypes.c_int]),
                       ("check_ffma_splits", [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
                       ("check_cl_split", []),
                       ("check_tail_schedule", [])):
        fn = getattr(lib, name)
        fn.argtypes = args + [ctypes.POINTER(ll)]
        fn.restype = ll
    return lib


def _run(fn, *args):
    n = ctypes.c_longlong(0)
    bad = fn(*args, ctypes.byref(n))
    return bad, n.value


def test_stream_k_ranges_partition_units(chk):
    bad, n = _run(chk.check_stream_k, 400, 160)
    assert n > 1_000_000 and bad == 0


def test_stream_k_ranges_near_int_limit(chk):
    bad, n = _run(chk.check_stream_k_large)
    assert n > 1000 and bad == 0


def test_weight_streaming_plan_matches_brute_force(chk):
    bad, n = _run(chk.check_sk_plan)
    assert n > 1000 and bad == 0


def test_tile_raster_is_a_banded_bijection(chk):
    bad, n = _run(chk.check_tile_coords, 40, 40)
    assert n > 100_000 and bad == 0


@pytest.mark.parametrize("num_sms", [148, 132, 1])
def test_fp32_split_k_ranges(chk, num_sms):
    bad, n = _run(chk.check_ffma_splits, 300, 600, num_sms)
    assert n > 100_000 and bad == 0


def test_cluster_split_plan(chk):
    bad, n = _run(chk.check_cl_split)
    assert n > 100_000 and bad == 0


def test_pair_kernel_tail_schedule(chk):
    bad, n = _run(chk.check_tail_schedule)
    assert n > 100_000 and bad == 0
