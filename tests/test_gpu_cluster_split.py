"""GPU parity of the weight-streaming kernel's split-K inside thread-block
clusters, against the fp64 oracle, through the C ABI.

With 16-bit weights, where T column groups times a split S in {8, 4, 2, 1}
fill at least three quarters of the SMs, the k-range of group t is split
over the S CTAs of one cluster and the partials meet in distributed shared
memory (each rank owns GN/S columns and sums the S partials in rank order);
other shapes keep stream-K.  The 16-bit shapes below are picked so that, on
a 148-SM device, every split and stream-K is taken (GN = 128 columns,
128-row k-units), each with ragged M, N and K.  4-bit weights always take
stream-K; the 4-bit shapes give it the same spread of group counts
(GN = 256, 64-row k-units).  The regular calls are held to the
weight-streaming kernel by a tuning rule.  Tolerances are those of the
plain parity tests; integer data must match bit-exactly (every partial sum
is exact, whatever the order), and repeated calls must agree bit for bit.
"""
import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth
from gpu_util import to_dev, from_dev, decode16, guarded_out, check_guard, assert_close, rel_frob

pytestmark = pytest.mark.gpu
RTOL = ATOL = 1e-2
FROB = {"f16": 2e-3, "bf16": 1e-2}

# (M, N, K): T = ceil(N / 128) groups, KB = ceil(K / 128) k-units
SHAPES16 = [(16, 2000, 1100),     # T 16: S = 8 (4 if 16 clusters of 8 do not fit)
            (7, 4000, 600),       # T 32: S = 4
            (33, 8000, 300),      # T 63: S = 2
            (100, 16000, 200),    # T 125: S = 1 (whole groups, no reduction)
            (16, 1000, 640)]      # T 8: stream-K
# (M, N, K): T = ceil(N / 256) groups, KB = K / 64 k-units (K multiple of
# 128); stream-K over 16, 32, 63, 118 and 4 groups
SHAPES4 = [(16, 4000, 640), (5, 8000, 384), (20, 16000, 256), (3, 30000, 128), (40, 1000, 512)]


@pytest.fixture(scope="module")
def tg():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_dense_gemm_tma_b200 as tg
    tg.load_library()
    yield tg
    tg.tune_set([])


@pytest.fixture
def small_m(tg):
    # every small-M call on the weight-streaming kernel, all SMs
    tg.tune_set([{"op": op, "path": "small_m", "m_lo": 1, "m_hi": 128}
                 for op in ("bf16", "f16", "w4a16", "wfp4")])
    yield
    tg.tune_set([])


def _run16(tg, kind, A, B, relu=False, tb=False):
    import torch
    M, K = A.shape
    N = B.shape[1]
    big, C, pad = guarded_out(M, N, kind)
    fn = tg.gemm_bf16 if kind == "bf16" else tg.gemm_f16
    Bs = np.ascontiguousarray(B.T) if tb else B
    fn(to_dev(A, kind), to_dev(Bs, kind), C=C, relu=relu, trans_b=tb)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    check_guard(big, kind, M, N, pad)
    return from_dev(C, kind)


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("shape", SHAPES16)
def test_16bit(tg, small_m, kind, shape):
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=5, dtype=kind, scale_by_sqrt_k=True)
    ref_fn = oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16
    for relu in (False, True):
        bits = _run16(tg, kind, A, B, relu)
        got = decode16(bits, kind)
        ref = ref_fn(A, B, relu)
        assert_close(got, ref, RTOL, ATOL, f"{kind} {shape} relu={relu}")
        assert rel_frob(got, ref) <= FROB[kind]
        assert np.array_equal(_run16(tg, kind, A, B, relu), bits), "repeat"


@pytest.mark.parametrize("shape", SHAPES16[:4])
def test_16bit_transposed_b(tg, shape):
    # B stored N x K: the kernel reads K-major weight tiles (no tuning rule
    # applies to transposed calls; small M takes this kernel by default)
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=6, dtype="bf16", scale_by_sqrt_k=True)
    got = decode16(_run16(tg, "bf16", A, B, tb=True), "bf16")
    ref = oracle.gemm_bf16(A, B, False)
    assert_close(got, ref, RTOL, ATOL, f"tb {shape}")
    assert rel_frob(got, ref) <= FROB["bf16"]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("shape", [SHAPES16[1], SHAPES16[2]])
def test_16bit_integer_bit_exact(tg, small_m, kind, shape):
    M, N, K = shape
    A, B = synth.integers(M, N, K, seed=1, lo=-1, hi=1, dtype=kind)
    got = _run16(tg, kind, A, B)
    ref = (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B)
    rnd = oracle.round_bf16(ref) if kind == "bf16" else oracle.round_f16(ref)
    assert np.array_equal(got, rnd)


def _run_w4(tg, A, Bq, S, N, relu=False):
    import torch
    M = A.shape[0]
    big, C, pad = guarded_out(M, N, "f16")
    tg.gemm_w4a16(to_dev(A, "f16"), to_dev(Bq, "u8"), to_dev(S, "f16"), N, C=C, relu=relu)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    check_guard(big, "f16", M, N, pad)
    return from_dev(C, "f16")


def _run_fp4(tg, A, Bq, E, N, relu=False):
    import torch
    M = A.shape[0]
    big, C, pad = guarded_out(M, N, "bf16")
    tg.gemm_wfp4(to_dev(A, "bf16"), to_dev(Bq, "u8"), to_dev(E, "u8"), N, C=C, relu=relu)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    check_guard(big, "bf16", M, N, pad)
    return from_dev(C, "bf16")


@pytest.mark.parametrize("shape", SHAPES4)
def test_w4a16(tg, small_m, shape):
    M, N, K = shape
    A, Bq, S, _ = synth.w4a16(M, N, K, seed=7)
    for relu in (False, True):
        bits = _run_w4(tg, A, Bq, S, N, relu)
        got = decode16(bits, "f16")
        ref = oracle.gemm_w4a16(A, Bq, S, N=N, relu=relu)
        assert_close(got, ref, RTOL, ATOL, f"w4a16 {shape} relu={relu}")
        assert rel_frob(got, ref) <= 2e-3
        assert np.array_equal(_run_w4(tg, A, Bq, S, N, relu), bits), "repeat"


@pytest.mark.parametrize("shape", SHAPES4)
def test_wfp4(tg, small_m, shape):
    M, N, K = shape
    K = K - 32 if K > 128 else K            # K need not be a multiple of 128 here
    A, Bq, E, _ = synth.wfp4(M, N, K, seed=8)
    for relu in (False, True):
        bits = _run_fp4(tg, A, Bq, E, N, relu)
        got = decode16(bits, "bf16")
        ref = oracle.gemm_wfp4(A, Bq, E, N=N, relu=relu)
        assert_close(got, ref, RTOL, ATOL, f"wfp4 {shape} relu={relu}")
        assert rel_frob(got, ref) <= 1e-2
        assert np.array_equal(_run_fp4(tg, A, Bq, E, N, relu), bits), "repeat"


def test_w4a16_power_of_two_scales_bit_exact(tg, small_m):
    # small integer activations and power-of-two scales: every product and
    # partial sum is exact, so the summation order cannot show
    M, N, K = 5, 8000, 384
    A, Bq, _, q = synth.w4a16(M, N, K, seed=9, a_int=1)
    rng = np.random.default_rng(9)
    S = synth.store(np.ldexp(1.0, rng.integers(-4, 0, size=(K // 128, N))), "f16")
    got = _run_w4(tg, A, Bq, S, N)
    ref = oracle.gemm_w4a16(A, Bq, S, N=N)
    assert np.array_equal(got, oracle.round_f16(ref))
