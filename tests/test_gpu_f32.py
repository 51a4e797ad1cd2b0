"""GPU parity of the fp32 FFMA path against the fp64 oracle, through the C ABI.

Tolerance: relative Frobenius error <= 1e-5 on random data; integer-valued
inputs ({-3..3}, |partial sums| < 2^24) must match bit-exactly.
"""
import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth
from gpu_util import to_dev, from_dev, guarded_out, check_guard, rel_frob

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tg():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_dense_gemm_tma_b200 as tg
    tg.load_library()
    return tg


def _run(tg, A, B, relu=False, guard=True):
    import torch
    M, K = A.shape
    N = B.shape[1]
    if guard:
        big, C, pad = guarded_out(M, N, "f32")
    else:
        C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    tg.gemm_f32(to_dev(A, "f32"), to_dev(B, "f32"), C=C, relu=relu, mode=tg.F32_FFMA)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    if guard:
        check_guard(big, "f32", M, N, pad)
    return from_dev(C, "f32")


def test_small_uniform_256(tg):
    A, B = synth.uniform_pm1(256, 256, 256, seed=0)
    got = _run(tg, A, B)
    assert rel_frob(got, oracle.gemm_f32(A, B)) <= 1e-5


@pytest.mark.parametrize("shape", [(1024, 1024, 1024), (300, 520, 200), (129, 127, 1001),
                                   (1, 1, 1), (7, 13, 33), (130, 260, 64)])
@pytest.mark.parametrize("relu", [False, True])
def test_normal_shapes(tg, shape, relu):
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=1)
    got = _run(tg, A, B, relu)
    ref = oracle.gemm_f32(A, B, relu)
    assert rel_frob(got, ref) <= 1e-5
    if relu:
        assert np.all(got >= 0)


def test_integer_bit_exact_1024(tg):
    A, B = synth.integers(1024, 1024, 1024, seed=1)
    got = _run(tg, A, B)
    assert np.array_equal(got, oracle.round_f32(oracle.gemm_f32(A, B)))
    got = _run(tg, A, B, relu=True)
    assert np.array_equal(got, oracle.round_f32(oracle.gemm_f32(A, B, relu=True)))


@pytest.mark.parametrize("kind", ["normal", "integer"])
def test_full_size_4096_sampled(tg, kind):
    n = 4096
    if kind == "normal":
        A, B = synth.normal(n, n, n, seed=1)
    else:
        A, B = synth.integers(n, n, n, seed=1)
    got = _run(tg, A, B, guard=False)
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 40, replace=False)]))
    cols = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 40, replace=False)]))
    ref_r = oracle.gemm_f32(np.ascontiguousarray(A[rows]), B)
    ref_c = oracle.gemm_f32(A, np.ascontiguousarray(B[:, cols]))
    if kind == "integer":
        assert np.array_equal(got[rows], oracle.round_f32(ref_r))
        assert np.array_equal(got[:, cols], oracle.round_f32(ref_c))
    else:
        assert rel_frob(got[rows], ref_r) <= 1e-5
        assert rel_frob(got[:, cols], ref_c) <= 1e-5


@pytest.mark.parametrize("shape", [(200, 200, 3000), (129, 127, 1001), (64, 1000, 4096)])
def test_split_k_shapes(tg, shape):
    # fewer 128 x 128 tiles than SMs: K is split over several CTAs per tile
    # (up to 8 ranges) and the partial tiles are added in range order
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=1)
    for relu in (False, True):
        got = _run(tg, A, B, relu)
        assert rel_frob(got, oracle.gemm_f32(A, B, relu)) <= 1e-5


def test_split_k_integer_bit_exact_and_repeatable(tg):
    A, B = synth.integers(100, 300, 2048, seed=1)
    got = _run(tg, A, B)
    assert np.array_equal(got, oracle.round_f32(oracle.gemm_f32(A, B)))
    A, B = synth.normal(1024, 1024, 1024, seed=1)
    first = _run(tg, A, B)
    for _ in range(3):
        assert np.array_equal(_run(tg, A, B), first)
