"""GPU parity of the dequantize GEMM (fp16 activations x signed 4-bit weights
with fp16 group scales) against the fp64 oracle, which dequantises
explicitly, through the C ABI.

Tolerance: rtol = atol = 1e-2 (the pages' check).  With power-of-two scales
and small integer activations every dequantised weight and every partial sum
is exact, so that case must match bit-exactly.
"""
import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth
from gpu_util import to_dev, from_dev, decode16, guarded_out, check_guard, assert_close, rel_frob

pytestmark = pytest.mark.gpu
RTOL = ATOL = 1e-2


@pytest.fixture(scope="module")
def tg():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_dense_gemm_tma_b200 as tg
    tg.load_library()
    return tg


def _run(tg, A, Bq, S, N, relu=False, guard=True):
    import torch
    M = A.shape[0]
    if guard:
        big, C, pad = guarded_out(M, N, "f16")
    else:
        C = None
    C = tg.gemm_w4a16(to_dev(A, "f16"), to_dev(Bq, "u8"), to_dev(S, "f16"), N, C=C, relu=relu)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    if guard:
        check_guard(big, "f16", M, N, pad)
    return decode16(from_dev(C, "f16"), "f16")


@pytest.mark.parametrize("shape", [(4, 256, 256), (130, 300, 384), (1, 64, 128), (257, 520, 640),
                                   (16, 8192, 1024), (64, 1000, 512), (33, 301, 256)])
@pytest.mark.parametrize("relu", [False, True])
def test_random(tg, shape, relu):
    M, N, K = shape
    A, Bq, S, _ = synth.w4a16(M, N, K, seed=4)
    got = _run(tg, A, Bq, S, N, relu)
    ref = oracle.gemm_w4a16(A, Bq, S, N=N, relu=relu)
    assert_close(got, ref, RTOL, ATOL, f"w4a16 {shape}")
    # relative Frobenius error at the fp16 output-rounding level
    assert rel_frob(got, ref) <= 2e-3


def test_bit_exact_power_of_two_scales(tg):
    M, N, K = 64, 512, 256
    A, Bq, _, q = synth.w4a16(M, N, K, seed=4, a_int=1)
    S = synth.store(np.full((K // 128, N), 0.125), "f16")
    got = _run(tg, A, Bq, S, N)
    ref = oracle.gemm_w4a16(A, Bq, S, N=N)
    assert np.array_equal(got, decode16(oracle.round_f16(ref), "f16"))


def test_group_boundaries(tg):
    # scales differ per group: a wrong group index shows up at once
    M, N, K = 8, 256, 512
    A, Bq, _, q = synth.w4a16(M, N, K, seed=5)
    S = synth.store(np.array([[0.25], [0.5], [1.0], [2.0]]) * np.ones((1, N)), "f16")
    got = _run(tg, A, Bq, S, N)
    ref = oracle.gemm_w4a16(A, Bq, S, N=N)
    assert_close(got, ref, RTOL, ATOL, "groups")
    assert rel_frob(got, ref) <= 2e-3


@pytest.mark.parametrize("M", [1, 16, 4096])
def test_full_size(tg, M):
    N = K = 8192
    A, Bq, S, _ = synth.w4a16(M, N, K, seed=4)
    got = _run(tg, A, Bq, S, N, guard=False)
    if M <= 16:
        ref = oracle.gemm_w4a16(A, Bq, S, N=N)
        assert_close(got, ref, RTOL, ATOL, f"M={M}")
        assert rel_frob(got, ref) <= 2e-3
    else:
        rng = np.random.default_rng(3)
        rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 24, replace=False)]))
        ref = oracle.gemm_w4a16(np.ascontiguousarray(A[rows]), Bq, S, N=N)
        assert_close(got[rows], ref, RTOL, ATOL, "rows")
        cols = np.arange(4096, 4096 + 256)
        ref_c = oracle.gemm_w4a16(A, np.ascontiguousarray(Bq[:, 2048:2048 + 128]),
                                  np.ascontiguousarray(S[:, 4096:4096 + 256]), N=256)
        assert_close(got[:, cols], ref_c, RTOL, ATOL, "cols")


def test_pair_kernel_repeatable(tg):
    # M > 128 runs on CTA pairs whose converter warps hand their half of each
    # weight slice to the other CTA's tensor core: repeated calls must agree
    # bit for bit (a missing ordering between the halves would show here)
    M, N, K = 1024, 2048, 2048
    A, Bq, S, _ = synth.w4a16(M, N, K, seed=4)
    first = _run(tg, A, Bq, S, N, guard=False)
    ref = oracle.gemm_w4a16(np.ascontiguousarray(A[:64]), Bq, S, N=N)
    assert_close(first[:64], ref, RTOL, ATOL, "pair rows 0..63")
    for _ in range(10):
        assert np.array_equal(_run(tg, A, Bq, S, N, guard=False), first)
