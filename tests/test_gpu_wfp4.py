"""GPU parity of the FP4-weight GEMM (bf16 activations x MXFP4 weights: E2M1
codes with one E8M0 scale per 32 k of a column) against the fp64 oracle,
which dequantises explicitly, through the C ABI (tg_gemm_wfp4).

Tolerance: rtol = atol = 1e-2 elementwise and relative Frobenius error
<= 1e-2 (the bf16 output's rounding), as for the bf16 GEMM.  Every random
case draws all 16 E2M1 codes.  With integer activations every product
a * e2m1 * 2^(E - 127) and every partial sum is exact in fp32 (the scales
chosen keep all terms on a grid of 2^-4 well inside 2^24), so the GPU's one
rounding of the exact sum to bf16 must equal the oracle's bit for bit; that
case varies the scale per 32-row block and per column, which pins the
block indexing and the converter's column order.  Shapes cover M <= 4, the
weight-streaming kernel (M <= 128), the CTA-pair kernel (M > 128), ragged
N (odd, not a multiple of the 256 columns a unit holds) and ragged K (not a
multiple of 32 or 64).
"""
import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth
from gpu_util import to_dev, from_dev, decode16, guarded_out, check_guard, assert_close, rel_frob

pytestmark = pytest.mark.gpu
RTOL = ATOL = 1e-2
FROB = 1e-2


@pytest.fixture(scope="module")
def tg():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_dense_gemm_tma_b200 as tg
    tg.load_library()
    return tg


def _run(tg, A, Bq, E, N, relu=False, guard=True):
    import torch
    M = A.shape[0]
    C = None
    if guard:
        big, C, pad = guarded_out(M, N, "bf16")
    C = tg.gemm_wfp4(to_dev(A, "bf16"), to_dev(Bq, "u8"), to_dev(E, "u8"), N, C=C, relu=relu)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    if guard:
        check_guard(big, "bf16", M, N, pad)
    return from_dev(C, "bf16")


SHAPES = [(1, 256, 256), (3, 301, 96), (16, 2048, 1024), (17, 520, 200), (64, 1000, 512),
          (128, 2304, 4096), (129, 300, 384), (257, 520, 640), (300, 777, 1000)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("relu", [False, True])
def test_random(tg, shape, relu):
    M, N, K = shape
    A, Bq, E, codes = synth.wfp4(M, N, K, seed=4)
    assert len(np.unique(codes)) == 16 or codes.size < 64
    got = decode16(_run(tg, A, Bq, E, N, relu), "bf16")
    ref = oracle.gemm_wfp4(A, Bq, E, N=N, relu=relu)
    assert_close(got, ref, RTOL, ATOL, f"wfp4 {shape} relu={relu}")
    assert rel_frob(got, ref) <= FROB
    if relu:
        assert np.all(got >= 0)


def _exact_case(M, N, K, seed):
    """Integer activations in {-2..2}, all codes, scales 2^-3 .. 2^2 varying
    per 32-row block and column: every sum exact in fp32."""
    A, Bq, _, codes = synth.wfp4(M, N, K, seed=seed, a_int=2)
    rng = np.random.default_rng(seed + 100)
    E = rng.integers(124, 130, size=((K + 31) // 32, N)).astype(np.uint8)
    return A, Bq, E


@pytest.mark.parametrize("shape", [(2, 520, 256), (24, 1000, 320), (300, 264, 224)])
def test_bit_exact_block_scales(tg, shape):
    M, N, K = shape
    A, Bq, E = _exact_case(M, N, K, seed=5)
    got = _run(tg, A, Bq, E, N)
    ref = oracle.gemm_wfp4(A, Bq, E, N=N)
    assert np.array_equal(decode16(got, "bf16"), decode16(oracle.round_bf16(ref), "bf16"))


def test_large_scale_exponents(tg):
    # E up to 140 (scales up to 2^13): the converter applies those with a
    # second exact multiply; small E (2^-20) checks the low end
    M, N, K = 40, 512, 256
    A, Bq, _, _ = synth.wfp4(M, N, K, seed=6)
    rng = np.random.default_rng(6)
    E = rng.integers(107, 141, size=(K // 32, N)).astype(np.uint8)
    got = decode16(_run(tg, A, Bq, E, N), "bf16")
    ref = oracle.gemm_wfp4(A, Bq, E, N=N)
    assert_close(got, ref, RTOL, ATOL * float(np.abs(ref).max()), "large E")
    assert rel_frob(got, ref) <= FROB
    # the same with integer activations is exact
    # (E <= 135: |sum| <= 2 * 6 * 2^8 * K stays within 24 bits of the 2^-2 grid)
    A, Bq, _ = _exact_case(M, N, K, seed=7)
    E = rng.integers(126, 136, size=(K // 32, N)).astype(np.uint8)
    got = _run(tg, A, Bq, E, N)
    ref = oracle.gemm_wfp4(A, Bq, E, N=N)
    assert np.array_equal(decode16(got, "bf16"), decode16(oracle.round_bf16(ref), "bf16"))


@pytest.mark.parametrize("M", [8, 300])
def test_nan_scale(tg, M):
    # an E8M0 byte of 255 is NaN: exactly the columns with such a block are NaN
    N, K = 264, 128
    A, Bq, E, _ = synth.wfp4(M, N, K, seed=8)
    E = E.copy()
    E[1, 5] = 255
    E[3, 200] = 255
    got = decode16(_run(tg, A, Bq, E, N), "bf16")
    ref = oracle.gemm_wfp4(A, Bq, E, N=N)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert set(np.where(np.isnan(got).any(axis=0))[0]) == {5, 200}
    ok = ~np.isnan(ref)
    assert_close(got[ok], ref[ok], RTOL, ATOL, "non-NaN columns")


@pytest.mark.parametrize("M", [1, 16, 4096])
def test_full_size(tg, M):
    N = K = 8192
    A, Bq, E, _ = synth.wfp4(M, N, K, seed=4)
    got = decode16(_run(tg, A, Bq, E, N, guard=False), "bf16")
    if M <= 16:
        ref = oracle.gemm_wfp4(A, Bq, E, N=N)
        assert_close(got, ref, RTOL, ATOL, f"M={M}")
        assert rel_frob(got, ref) <= FROB
    else:
        rng = np.random.default_rng(3)
        rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 24, replace=False)]))
        ref = oracle.gemm_wfp4(np.ascontiguousarray(A[rows]), Bq, E, N=N)
        assert_close(got[rows], ref, RTOL, ATOL, "rows")
        assert rel_frob(got[rows], ref) <= FROB
        cols = np.arange(4096, 4096 + 256)
        ref_c = oracle.gemm_wfp4(A, np.ascontiguousarray(Bq[:, 2048:2048 + 128]),
                                 np.ascontiguousarray(E[:, 4096:4096 + 256]), N=256)
        assert_close(got[:, cols], ref_c, RTOL, ATOL, "cols")
        assert rel_frob(got[:, cols], ref_c) <= FROB


def test_repeatable(tg):
    # the CTA-pair kernel's converters hand half of each weight slice to the
    # other CTA's tensor cores, and the small-M kernel sums split-K partials
    # in a fixed order: repeated calls agree bit for bit
    for M, N, K in ((1024, 2048, 2048), (16, 4096, 8192)):
        A, Bq, E, _ = synth.wfp4(M, N, K, seed=4)
        first = _run(tg, A, Bq, E, N, guard=False)
        for _ in range(5):
            assert np.array_equal(_run(tg, A, Bq, E, N, guard=False), first)


def test_k_zero_and_empty(tg):
    import torch
    A = torch.empty((5, 0), dtype=torch.bfloat16, device="cuda")
    Bq = torch.empty((0, 16), dtype=torch.uint8, device="cuda")
    E = torch.empty((0, 32), dtype=torch.uint8, device="cuda")
    big, C, pad = guarded_out(5, 24, "bf16")
    tg.gemm_wfp4(A, Bq, E, 24, C=C)
    torch.cuda.synchronize()
    assert np.all(from_dev(C, "bf16") == 0)
    check_guard(big, "bf16", 5, 24, pad)
