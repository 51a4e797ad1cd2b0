"""tg_gemm_bf16_small_m_static: the small-M bf16 GEMM for callers that must
not allocate device memory (its split-K scratch is a fixed device array in
the library).  Called through the C ABI and compared with tg_gemm_bf16, the
regular entry point, on two calls in a row; also checks the size limit.

This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

from tiled_dense_gemm_tma_b200 import synth
from gpu_util import to_dev, from_dev, decode16, guarded_out, check_guard, assert_close

pytestmark = pytest.mark.gpu
RTOL = ATOL = 1e-2          # the tolerance of the bf16 parity tests
TG_OK, TG_ERR_UNSUPPORTED = 0, 3


@pytest.fixture(scope="module")
def lib():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_dense_gemm_tma_b200 as tg
    return tg.load_library()


def _call(lib, fn_name, A, B, C, relu):
    import torch
    M, K = A.shape
    N = B.shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return getattr(lib, fn_name)(M, N, K, A.data_ptr(), A.stride(0), B.data_ptr(), B.stride(0),
                                 C.data_ptr(), C.stride(0), 1 if relu else 0, stream)


@pytest.mark.parametrize("shape,relu", [((16, 4096, 4096), False), ((100, 777, 1200), True),
                                        ((1, 2048, 640), False), ((128, 2304, 4096), False)])
def test_matches_regular_entry_point_twice(lib, shape, relu):
    import torch
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=3, dtype="bf16", scale_by_sqrt_k=True)
    dA, dB = to_dev(A, "bf16"), to_dev(B, "bf16")
    big_ref, C_ref, pad = guarded_out(M, N, "bf16")
    assert _call(lib, "tg_gemm_bf16", dA, dB, C_ref, relu) == TG_OK
    torch.cuda.synchronize()
    ref = decode16(from_dev(C_ref, "bf16"), "bf16")
    for _ in range(2):
        big, C, pad = guarded_out(M, N, "bf16")
        assert _call(lib, "tg_gemm_bf16_small_m_static", dA, dB, C, relu) == TG_OK
        torch.cuda.synchronize()
        assert lib.tg_last_device_status(None) == TG_OK
        check_guard(big, "bf16", M, N, pad)
        got = decode16(from_dev(C, "bf16"), "bf16")
        assert_close(got, ref, RTOL, ATOL, f"static {shape}")


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
