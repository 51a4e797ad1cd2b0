"""GPU parity of the tensor-core paths (fp16, bf16, TF32 mode) against the
fp64 oracle, called through the C ABI (ctypes binding).

Tolerances: fp16 / bf16 use rtol = atol = 1e-2 (assert_close semantics, the
pages' check); TF32 mode uses relative Frobenius error <= 5e-3; integer
valued inputs must match bit-exactly.  Every output is written into a guard-
banded buffer whose margin must stay untouched.
"""
import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth
from gpu_util import (to_dev, from_dev, decode16, guarded_out, check_guard, assert_close,
                      rel_frob)

pytestmark = pytest.mark.gpu

RTOL = ATOL = 1e-2
# stricter diagnostic bounds on relative Frobenius error for N(0,1)/sqrt(K) data
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


def _oracle16(kind, A, B, relu=False):
    return (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B, relu)


SHAPES = [(256, 256, 256), (300, 520, 200), (129, 127, 1000), (1, 1, 1), (7, 13, 69),
          (128, 256, 64), (640, 264, 130)]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("relu", [False, True])
def test_random_shapes(tg, kind, shape, relu):
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=2, dtype=kind, scale_by_sqrt_k=True)
    got = decode16(_run16(tg, kind, A, B, relu), kind)
    ref = _oracle16(kind, A, B, relu)
    assert_close(got, ref, RTOL, ATOL, f"{kind} {shape} relu={relu}")
    assert rel_frob(got, ref) <= FROB[kind]
    if relu:
        assert np.all(got >= 0)


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_integer_inputs_bit_exact(tg, kind):
    # {-1, 0, 1} entries, K = 256: every partial sum is an integer of
    # magnitude <= 256, exact in fp32 and in the 16-bit output.
    M, N, K = 200, 300, 256
    A, B = synth.integers(M, N, K, seed=1, lo=-1, hi=1, dtype=kind)
    got = _run16(tg, kind, A, B)
    ref = _oracle16(kind, A, B)
    rnd = oracle.round_bf16(ref) if kind == "bf16" else oracle.round_f16(ref)
    assert np.array_equal(got, rnd)
    got_r = _run16(tg, kind, A, B, relu=True)
    ref_r = _oracle16(kind, A, B, relu=True)
    rnd_r = oracle.round_bf16(ref_r) if kind == "bf16" else oracle.round_f16(ref_r)
    # relu of an exact negative gives +0 or -0; compare numerically
    assert np.array_equal(decode16(got_r, kind), decode16(rnd_r, kind))


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_multi_tile_1024(tg, kind):
    A, B = synth.normal(1024, 1024, 1024, seed=2, dtype=kind, scale_by_sqrt_k=True)
    got = decode16(_run16(tg, kind, A, B), kind)
    ref = _oracle16(kind, A, B)
    assert_close(got, ref, RTOL, ATOL, kind)
    assert rel_frob(got, ref) <= FROB[kind]


def test_k_zero_writes_zeros(tg):
    import torch
    A = torch.empty((5, 0), dtype=torch.bfloat16, device="cuda")
    B = torch.empty((0, 24), dtype=torch.bfloat16, device="cuda")
    big, C, pad = guarded_out(5, 24, "bf16")
    tg.gemm_bf16(A, B, C=C)
    torch.cuda.synchronize()
    assert np.all(from_dev(C, "bf16") == 0)
    check_guard(big, "bf16", 5, 24, pad)


def _sampled_check(tg, kind, M, N, K, seed, relu=False, nsamp=48):
    """Full-size run; check sampled full rows and full columns against the oracle."""
    import torch
    A, B = synth.normal(M, N, K, seed=seed, dtype=kind, scale_by_sqrt_k=True)
    fn = tg.gemm_bf16 if kind == "bf16" else tg.gemm_f16
    C = fn(to_dev(A, kind), to_dev(B, kind), relu=relu)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    got = decode16(from_dev(C, kind), kind)
    rng = np.random.default_rng(99)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, nsamp, replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, nsamp, replace=False)]))
    ref_rows = _oracle16(kind, np.ascontiguousarray(A[rows]), B, relu)
    assert_close(got[rows], ref_rows, RTOL, ATOL, f"{kind} rows")
    ref_cols = _oracle16(kind, A, np.ascontiguousarray(B[:, cols]), relu)
    assert_close(got[:, cols], ref_cols, RTOL, ATOL, f"{kind} cols")
    # the relative Frobenius gate is the sharp one (|C| ~ 1e-2 with these
    # entries): it covers every sampled row and every sampled column
    assert rel_frob(got[rows], ref_rows) <= FROB[kind]
    assert rel_frob(got[:, cols], ref_cols) <= FROB[kind]
    if relu:
        assert np.all(got[rows] >= 0) and np.all(got[:, cols] >= 0)


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("size", [4096, 8192])
@pytest.mark.parametrize("relu", [False, True])
def test_full_size_square_sampled(tg, kind, size, relu):
    _sampled_check(tg, kind, size, size, size, seed=2, relu=relu)


@pytest.mark.parametrize("shape", [(8192, 1024, 8192), (3000, 5000, 4000), (128, 14336, 4096),
                                   (16, 8192, 8192)])
def test_bf16_skinny_sampled(tg, shape):
    M, N, K = shape
    _sampled_check(tg, "bf16", M, N, K, seed=3, nsamp=min(48, M - 2))


# ------------------------------------------------------------------ TF32 mode

def _run_f32(tg, A, B, mode, relu=False):
    import torch
    M, K = A.shape
    N = B.shape[1]
    big, C, pad = guarded_out(M, N, "f32")
    tg.gemm_f32(to_dev(A, "f32"), to_dev(B, "f32"), C=C, relu=relu, mode=mode)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    check_guard(big, "f32", M, N, pad)
    return from_dev(C, "f32")


@pytest.mark.parametrize("shape", [(512, 768, 384), (300, 520, 200), (1, 1, 1), (129, 127, 1000)])
def test_tf32_random(tg, shape):
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=1)
    got = _run_f32(tg, A, B, tg.F32_TF32)
    ref = oracle.gemm_f32(A, B)
    assert rel_frob(got, ref) <= 5e-3


def test_tf32_full_1024(tg):
    # the TF32 configuration at 1024^3, every output against the oracle
    A, B = synth.normal(1024, 1024, 1024, seed=1)
    got = _run_f32(tg, A, B, tg.F32_TF32)
    assert rel_frob(got, oracle.gemm_f32(A, B)) <= 5e-3


def test_tf32_many_tiles_per_cta(tg):
    # 16 x 29 = 464 tiles of 128 x 256 for 148 persistent CTAs (> 3 per CTA):
    # every CTA wraps both TMEM accumulator buffers and the ring phases
    # several times; ragged N and K
    M, N, K = 2048, 7400, 100
    A, B = synth.normal(M, N, K, seed=1)
    for relu in (False, True):
        got = _run_f32(tg, A, B, tg.F32_TF32, relu=relu)
        assert rel_frob(got, oracle.gemm_f32(A, B, relu)) <= 5e-3


@pytest.mark.parametrize("kind", ["normal", "integer"])
def test_tf32_full_size_4096_sampled(tg, kind):
    # the TF32 configuration at 4096^3 (512 tiles): sampled full rows and
    # columns; integer data {-3..3} is exact in TF32 and fp32, so bit-exact
    import torch
    n = 4096
    A, B = synth.normal(n, n, n, seed=1) if kind == "normal" else synth.integers(n, n, n, seed=1)
    C = tg.gemm_f32(to_dev(A, "f32"), to_dev(B, "f32"), mode=tg.F32_TF32)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    got = from_dev(C, "f32")
    rng = np.random.default_rng(11)
    rows = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 40, replace=False)]))
    cols = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 40, replace=False)]))
    ref_r = oracle.gemm_f32(np.ascontiguousarray(A[rows]), B)
    ref_c = oracle.gemm_f32(A, np.ascontiguousarray(B[:, cols]))
    if kind == "integer":
        assert np.array_equal(got[rows], oracle.round_f32(ref_r))
        assert np.array_equal(got[:, cols], oracle.round_f32(ref_c))
    else:
        assert rel_frob(got[rows], ref_r) <= 5e-3
        assert rel_frob(got[:, cols], ref_c) <= 5e-3


def test_tf32_integer_bit_exact(tg):
    A, B = synth.integers(256, 384, 1024, seed=1)
    got = _run_f32(tg, A, B, tg.F32_TF32)
    assert np.array_equal(got, oracle.round_f32(oracle.gemm_f32(A, B)))
    got = _run_f32(tg, A, B, tg.F32_TF32, relu=True)
    assert np.array_equal(got, oracle.round_f32(oracle.gemm_f32(A, B, relu=True)))


@pytest.mark.parametrize("shape", [(512, 768, 384), (129, 127, 1000), (2048, 7400, 100)])
def test_tf32_one_cta_forced(tg, shape):
    # TF32 with M > 128 runs on CTA pairs; the one-CTA kernel (M <= 128, and
    # the path when a cluster launch is refused) forced by a tuning rule,
    # including more tiles than CTAs (2048 x 7400: 464 tiles of 128 x 256)
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=1)
    tg.tune_set([{"op": "f32_tf32", "path": "one_cta"}])
    try:
        for relu in (False, True):
            got = _run_f32(tg, A, B, tg.F32_TF32, relu=relu)
            assert rel_frob(got, oracle.gemm_f32(A, B, relu)) <= 5e-3
        Ai, Bi = synth.integers(M, N, K, seed=1)
        got = _run_f32(tg, Ai, Bi, tg.F32_TF32)
        assert np.array_equal(got, oracle.round_f32(oracle.gemm_f32(Ai, Bi)))
    finally:
        tg.tune_set([])


def test_tf32_pair_forced_small_m(tg):
    # a CTA-pair rule for M <= 128: the partner CTA of every pair has no rows
    A, B = synth.integers(100, 1000, 520, seed=2)
    tg.tune_set([{"op": "f32_tf32", "path": "cta_pair"}])
    try:
        got = _run_f32(tg, A, B, tg.F32_TF32)
        assert np.array_equal(got, oracle.round_f32(oracle.gemm_f32(A, B)))
    finally:
        tg.tune_set([])


# ------------------------------------------- small M: weight-streaming kernel

SKINNY = [(1, 1000, 640), (2, 384, 4096), (16, 2048, 1000), (17, 520, 333), (33, 1024, 2048),
          (64, 130, 64), (65, 4096, 512), (100, 777, 1200), (128, 2304, 4096)]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("shape", SKINNY)
def test_skinny_shapes(tg, kind, shape):
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=3, dtype=kind, scale_by_sqrt_k=True)
    for relu in (False, True):
        got = decode16(_run16(tg, kind, A, B, relu), kind)
        ref = _oracle16(kind, A, B, relu)
        assert_close(got, ref, RTOL, ATOL, f"{kind} {shape} relu={relu}")
        assert rel_frob(got, ref) <= FROB[kind]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_skinny_integer_bit_exact_and_repeatable(tg, kind):
    # split-K partials are summed in a fixed order: bit-exact on integer data
    # and identical across repeated calls on random data
    M, N, K = 24, 1536, 256
    A, B = synth.integers(M, N, K, seed=1, lo=-1, hi=1, dtype=kind)
    got = _run16(tg, kind, A, B)
    ref = _oracle16(kind, A, B)
    rnd = oracle.round_bf16(ref) if kind == "bf16" else oracle.round_f16(ref)
    assert np.array_equal(got, rnd)
    A, B = synth.normal(16, 4096, 8192, seed=3, dtype=kind, scale_by_sqrt_k=True)
    first = _run16(tg, kind, A, B)
    for _ in range(3):
        assert np.array_equal(_run16(tg, kind, A, B), first)
