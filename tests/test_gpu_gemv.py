"""GPU parity of the CUDA-core path for one to four activation rows (M <= 4:
bf16, fp16 and 4-bit weights) against the fp64 oracle, through the C ABI.

Shapes cover ragged column tails (N not a multiple of the 256 or 512
columns a CTA owns, odd N for packed weights), ragged K (not a multiple of
the 128-row groups), K long enough to be split over several CTAs (partials
summed in a cluster through distributed shared memory, or by the last CTA
of a column block under stream-K), ReLU, and the bit-exact cases:
integer data in {-1, 0, 1} (16-bit weights) and power-of-two scales with
integer activations (4-bit weights).  Repeated calls must agree bit for bit
(the split-K partials are summed in a fixed order).
"""
import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth
from gpu_util import to_dev, from_dev, decode16, guarded_out, check_guard, assert_close, rel_frob

pytestmark = pytest.mark.gpu
RTOL = ATOL = 1e-2
FROB = {"f16": 2e-3, "bf16": 1e-2}


@pytest.fixture(scope="module")
def tg():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_dense_gemm_tma_b200 as tg
    tg.load_library()
    return tg


def _run16(tg, kind, A, B, relu=False):
    import torch
    M, K = A.shape
    N = B.shape[1]
    big, C, pad = guarded_out(M, N, kind)
    fn = tg.gemm_bf16 if kind == "bf16" else tg.gemm_f16
    fn(to_dev(A, kind), to_dev(B, kind), C=C, relu=relu)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    check_guard(big, kind, M, N, pad)
    return from_dev(C, kind)


def _run4(tg, A, Bq, S, N, relu=False):
    import torch
    M = A.shape[0]
    big, C, pad = guarded_out(M, N, "f16")
    tg.gemm_w4a16(to_dev(A, "f16"), to_dev(Bq, "u8"), to_dev(S, "f16"), N, C=C, relu=relu)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    check_guard(big, "f16", M, N, pad)
    return from_dev(C, "f16")


def _runfp4(tg, A, Bq, E, N, relu=False):
    import torch
    M = A.shape[0]
    big, C, pad = guarded_out(M, N, "bf16")
    tg.gemm_wfp4(to_dev(A, "bf16"), to_dev(Bq, "u8"), to_dev(E, "u8"), N, C=C, relu=relu)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    check_guard(big, "bf16", M, N, pad)
    return from_dev(C, "bf16")


SHAPES16 = [(1, 1, 1), (1, 8, 127), (2, 255, 129), (3, 257, 2048), (4, 1000, 5000),
            (1, 4104, 300), (4, 8192, 1024), (2, 520, 8192)]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("shape", SHAPES16)
def test_gemv_16bit(tg, kind, shape):
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=3, dtype=kind, scale_by_sqrt_k=True)
    for relu in (False, True):
        got = decode16(_run16(tg, kind, A, B, relu), kind)
        ref = (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B, relu)
        assert_close(got, ref, RTOL, ATOL, f"{kind} {shape} relu={relu}")
        assert rel_frob(got, ref) <= FROB[kind]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_gemv_16bit_integer_bit_exact_and_repeatable(tg, kind):
    M, N, K = 3, 1000, 256
    A, B = synth.integers(M, N, K, seed=1, lo=-1, hi=1, dtype=kind)
    got = _run16(tg, kind, A, B)
    ref = (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B)
    rnd = oracle.round_bf16(ref) if kind == "bf16" else oracle.round_f16(ref)
    assert np.array_equal(decode16(got, kind), decode16(rnd, kind))
    A, B = synth.normal(4, 4096, 8192, seed=3, dtype=kind, scale_by_sqrt_k=True)
    first = _run16(tg, kind, A, B)
    for _ in range(3):
        assert np.array_equal(_run16(tg, kind, A, B), first)


SHAPES4 = [(1, 30, 128), (2, 33, 384), (3, 511, 256), (4, 513, 2560), (1, 1000, 8192),
           (4, 4096, 1024), (2, 8192, 640)]


@pytest.mark.parametrize("shape", SHAPES4)
@pytest.mark.parametrize("relu", [False, True])
def test_gemv_w4a16(tg, shape, relu):
    M, N, K = shape
    A, Bq, S, _ = synth.w4a16(M, N, K, seed=4)
    got = decode16(_run4(tg, A, Bq, S, N, relu), "f16")
    ref = oracle.gemm_w4a16(A, Bq, S, N=N, relu=relu)
    assert_close(got, ref, RTOL, ATOL, f"w4a16 {shape} relu={relu}")
    assert rel_frob(got, ref) <= 2e-3


def test_gemv_w4a16_bit_exact_groups_and_repeatable(tg):
    # power-of-two scales, integer activations: every product, group sum and
    # scaled sum is exact
    M, N, K = 2, 1000, 512
    A, Bq, _, _ = synth.w4a16(M, N, K, seed=4, a_int=1)
    S = synth.store(np.array([[0.125], [0.25], [0.5], [1.0]]) * np.ones((1, N)), "f16")
    got = _run4(tg, A, Bq, S, N)
    ref = oracle.gemm_w4a16(A, Bq, S, N=N)
    assert np.array_equal(decode16(got, "f16"), decode16(oracle.round_f16(ref), "f16"))
    A, Bq, S, _ = synth.w4a16(1, 8192, 8192, seed=4)
    first = _run4(tg, A, Bq, S, 8192)
    for _ in range(3):
        assert np.array_equal(_run4(tg, A, Bq, S, 8192), first)


CLUSTER_SHAPES = [(1, 8000, 1280), (3, 8192, 640), (4, 4000, 1024), (2, 8192, 8192)]


@pytest.mark.parametrize("kind", ["w4a16", "wfp4", "bf16", "f16"])
@pytest.mark.parametrize("shape", CLUSTER_SHAPES)
def test_gemv_cluster_and_stream_k_splits(tg, kind, shape):
    # These shapes give T column groups x a split S of 2 to 8 that fill the
    # GPU, so by default a group's k-range is split inside a cluster and the
    # partials meet in distributed shared memory (ragged N, a k-range of 5
    # units over 4 ranks, ragged K for 16-bit weights).  Capping the grid at
    # 100 CTAs leaves no such split and forces stream-K.  Both match the
    # oracle; each is repeatable bit for bit.
    M, N, K = shape
    if kind == "w4a16":
        A, Bq, S, _ = synth.w4a16(M, N, K, seed=5)
        ref = oracle.gemm_w4a16(A, Bq, S, N=N, relu=True)
        run = lambda: _run4(tg, A, Bq, S, N, relu=True)
        frob = 2e-3
    elif kind == "wfp4":
        A, Bq, E, _ = synth.wfp4(M, N, K, seed=5)
        ref = oracle.gemm_wfp4(A, Bq, E, N=N, relu=True)
        run = lambda: _runfp4(tg, A, Bq, E, N, relu=True)
        frob = FROB["bf16"]
    else:
        K = K - 24                                   # ragged in K
        A, B = synth.normal(M, N, K, seed=5, dtype=kind, scale_by_sqrt_k=True)
        ref = (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B, True)
        run = lambda: _run16(tg, kind, A, B, relu=True)
        frob = FROB[kind]
    for ctas in (0, 100):
        if ctas:
            tg.tune_set([{"op": kind, "path": "cuda_core", "m_lo": 1, "m_hi": 4, "ctas": ctas}])
        try:
            first = run()
            again = run()
        finally:
            tg.tune_set([])
        assert np.array_equal(first, again)
        got = decode16(first, {"w4a16": "f16", "wfp4": "bf16"}.get(kind, kind))
        assert_close(got, ref, RTOL, ATOL, f"{kind} {shape} ctas={ctas}")
        assert rel_frob(got, ref) <= frob


SHAPESFP4 = [(1, 256, 256), (2, 301, 96), (3, 520, 200), (4, 1000, 544), (1, 4104, 300),
             (2, 8192, 1024)]


@pytest.mark.parametrize("shape", SHAPESFP4)
@pytest.mark.parametrize("relu", [False, True])
def test_gemv_wfp4(tg, shape, relu):
    # FP4 weights (E2M1 codes, one E8M0 scale per 32 rows and column) on the
    # CUDA-core kernel: ragged N (odd, not a multiple of 256), K not a
    # multiple of the 32-row block or of the 256-row unit
    M, N, K = shape
    A, Bq, E, _ = synth.wfp4(M, N, K, seed=6)
    got = decode16(_runfp4(tg, A, Bq, E, N, relu), "bf16")
    ref = oracle.gemm_wfp4(A, Bq, E, N=N, relu=relu)
    assert_close(got, ref, RTOL, ATOL, f"wfp4 {shape} relu={relu}")
    assert rel_frob(got, ref) <= FROB["bf16"]


@pytest.mark.parametrize("M", [1, 3, 4])
def test_gemv_wfp4_bit_exact_scales_and_repeatable(tg, M):
    # integer activations in {-2..2} and every code: with scales 2^-3 .. 2^2
    # every partial sum is a multiple of 2^-4 below 2^14, and with the
    # smallest scales (E = 0, the subnormal 2^-127; E = 1, 2) a multiple of
    # 2^-128 below 2^-113: exact in fp32 either way, so C is the exact result
    # rounded once to bf16 (a subnormal bf16 in the second case)
    N, K = 1000, 320
    A, Bq, _, _ = synth.wfp4(M, N, K, seed=7, a_int=2)
    rng = np.random.default_rng(7)
    for lo, hi in ((124, 130), (0, 3)):
        E = rng.integers(lo, hi, size=((K + 31) // 32, N)).astype(np.uint8)
        got = _runfp4(tg, A, Bq, E, N)
        ref = oracle.gemm_wfp4(A, Bq, E, N=N)
        assert np.array_equal(decode16(got, "bf16"), decode16(oracle.round_bf16(ref), "bf16")), (lo, hi)
    A, Bq, E, _ = synth.wfp4(M, 8192, 8192, seed=4)
    first = _runfp4(tg, A, Bq, E, 8192)
    for _ in range(3):
        assert np.array_equal(_runfp4(tg, A, Bq, E, 8192), first)


@pytest.mark.parametrize("M", [1, 3])
def test_gemv_wfp4_nan_scale(tg, M):
    # an E8M0 byte of 255 is NaN: exactly the columns with such a block are NaN
    N, K = 264, 128
    A, Bq, E, _ = synth.wfp4(M, N, K, seed=8)
    E = E.copy()
    E[1, 5] = 255
    E[3, 200] = 255
    got = decode16(_runfp4(tg, A, Bq, E, N), "bf16")
    ref = oracle.gemm_wfp4(A, Bq, E, N=N)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert set(np.where(np.isnan(got).any(axis=0))[0]) == {5, 200}
    ok = ~np.isnan(ref)
    assert_close(got[ok], ref[ok], RTOL, ATOL, "non-NaN columns")
