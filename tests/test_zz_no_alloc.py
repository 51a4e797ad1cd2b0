"""tg_gemm_bf16_small_m_static: the small-M bf16 GEMM for callers that cannot
allocate device memory where they run it -- a program whose memory pool
already holds the device's free memory, or a loop that must stay out of the
driver's allocator.  Its split-K scratch is a fixed device array inside the
library, so no call allocates.

Called through the C ABI on two calls in a row and checked three ways:
against the fp64 oracle at the bf16 tolerance (rtol = atol = 1e-2, relative
Frobenius error <= 1e-2); against tg_gemm_bf16 bit for bit where both run
the same weight-streaming kernel with the same plan (5 <= M <= 128, the
regular call held to the small-M kernel on all SMs by a tuning rule: same
summation order), and within the tolerance where tg_gemm_bf16 takes its
CUDA-core kernel (M <= 4); and that a call on a stream the library has never seen
leaves the device's free memory unchanged.  Also checks the size limits.

This file is named to be collected last, so that a run stopping at the
first failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth
from gpu_util import (to_dev, from_dev, decode16, guarded_out, check_guard, assert_close,
                      rel_frob)

pytestmark = pytest.mark.gpu
RTOL = ATOL = 1e-2          # the tolerance of the bf16 parity tests
FROB = 1e-2
TG_OK, TG_ERR_UNSUPPORTED = 0, 3


@pytest.fixture(scope="module")
def lib():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_dense_gemm_tma_b200 as tg
    return tg.load_library()


def _call(lib, fn_name, A, B, C, relu, stream=None):
    import torch
    M, K = A.shape
    N = B.shape[1]
    s = stream if stream is not None else torch.cuda.current_stream()
    return getattr(lib, fn_name)(M, N, K, A.data_ptr(), A.stride(0), B.data_ptr(), B.stride(0),
                                 C.data_ptr(), C.stride(0), 1 if relu else 0,
                                 ctypes.c_void_p(s.cuda_stream))


@pytest.mark.parametrize("shape,relu", [((16, 4096, 4096), False), ((100, 777, 1200), True),
                                        ((1, 2048, 640), False), ((3, 1000, 700), True),
                                        ((5, 520, 333), False), ((128, 2304, 4096), False),
                                        ((64, 8192, 8192), True)])
def test_matches_oracle_and_regular_entry_point_twice(lib, shape, relu):
    import torch
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=3, dtype="bf16", scale_by_sqrt_k=True)
    ref = oracle.gemm_bf16(A, B, relu)
    dA, dB = to_dev(A, "bf16"), to_dev(B, "bf16")
    _, C_reg, _ = guarded_out(M, N, "bf16")
    # the regular call on the small-M kernel with its default plan (all SMs),
    # whatever the tuning table would choose for this shape
    import tiled_dense_gemm_tma_b200 as tg
    tg.tune_set([{"op": "bf16", "path": "small_m", "m_lo": 5, "m_hi": 128}] if M >= 5 else [])
    try:
        assert _call(lib, "tg_gemm_bf16", dA, dB, C_reg, relu) == TG_OK
        torch.cuda.synchronize()
    finally:
        tg.tune_set([])
    regular = from_dev(C_reg, "bf16")
    for _ in range(2):
        big, C, pad = guarded_out(M, N, "bf16")
        assert _call(lib, "tg_gemm_bf16_small_m_static", dA, dB, C, relu) == TG_OK
        torch.cuda.synchronize()
        assert lib.tg_last_device_status(None) == TG_OK
        check_guard(big, "bf16", M, N, pad)
        bits = from_dev(C, "bf16")
        got = decode16(bits, "bf16")
        assert_close(got, ref, RTOL, ATOL, f"static vs oracle {shape}")
        assert rel_frob(got, ref) <= FROB
        if M >= 5:
            # the same kernel, plan and summation order as tg_gemm_bf16
            assert np.array_equal(bits, regular), f"static vs tg_gemm_bf16 {shape}"
        else:
            assert_close(got, decode16(regular, "bf16"), RTOL, ATOL, f"static vs regular {shape}")


def test_allocates_nothing_on_a_new_stream(lib):
    import torch
    M, N, K = 32, 4096, 4096
    A, B = synth.normal(M, N, K, seed=3, dtype="bf16", scale_by_sqrt_k=True)
    dA, dB = to_dev(A, "bf16"), to_dev(B, "bf16")
    C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    # one call first: the array's device address is looked up on a device's
    # first call, which may also make the runtime load that part of the library
    assert _call(lib, "tg_gemm_bf16_small_m_static", dA, dB, C, False) == TG_OK
    torch.cuda.synchronize()
    first = from_dev(C, "bf16")
    fresh = torch.cuda.Stream()          # never used by tg_gemm_bf16: no workspace exists for it
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        assert _call(lib, "tg_gemm_bf16_small_m_static", dA, dB, C, False, stream=fresh) == TG_OK
    fresh.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert free_after == free_before, (free_before, free_after)
    assert lib.tg_last_device_status(None) == TG_OK
    assert np.array_equal(from_dev(C, "bf16"), first)


def test_rejects_sizes_beyond_the_scratch(lib):
    import torch
    # M = 128, N = 65536: 512 tiles of partials need far more than 16 MiB
    M, N, K = 128, 65536, 1024
    A = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((K, N), dtype=torch.bfloat16, device="cuda")
    C = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    assert _call(lib, "tg_gemm_bf16_small_m_static", A, B, C, False) == TG_ERR_UNSUPPORTED
    A2 = torch.zeros((129, 64), dtype=torch.bfloat16, device="cuda")
    B2 = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    C2 = torch.zeros((129, 64), dtype=torch.bfloat16, device="cuda")
    assert _call(lib, "tg_gemm_bf16_small_m_static", A2, B2, C2, False) == TG_ERR_UNSUPPORTED
