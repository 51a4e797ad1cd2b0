"""GPU parity of the 16-bit GEMM with transposed operands, C = op(A) . op(B)
(tg_gemm_f16_ex / tg_gemm_bf16_ex), and of the differentiable matmul built
on them (dA = dC . B^T, dB = A^T . dC), against the fp64 oracle.

The oracle multiplies the logical (untransposed) matrices; the GPU reads the
stored transposes.  Tolerance rtol = atol = 1e-2 as for the plain 16-bit
GEMM; integer data in {-1, 0, 1} must match bit-exactly.  Shapes include
ragged edges in every dimension, M below the 256-row pair tile, more pair
tiles than CTA pairs, and small M with B transposed (the weight-streaming
kernel on K-major weight tiles, or the CTA-pair kernel where the tuning rule
picks it).
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


def _run(tg, kind, A, B, ta, tb, relu=False):
    """A (M x K) and B (K x N) logical; pass the stored transposes."""
    import torch
    M, K = A.shape
    N = B.shape[1]
    As = np.ascontiguousarray(A.T) if ta else A
    Bs = np.ascontiguousarray(B.T) if tb else B
    big, C, pad = guarded_out(M, N, kind)
    fn = tg.gemm_bf16 if kind == "bf16" else tg.gemm_f16
    fn(to_dev(As, kind), to_dev(Bs, kind), C=C, relu=relu, trans_a=ta, trans_b=tb)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    check_guard(big, kind, M, N, pad)
    return from_dev(C, kind)


SHAPES = [(300, 520, 200), (129, 257, 1000), (64, 130, 72), (1024, 512, 256)]
TRANS = [(True, False), (False, True), (True, True)]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("trans", TRANS)
def test_transposed_operands(tg, kind, shape, trans):
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=2, dtype=kind, scale_by_sqrt_k=True)
    ref_fn = oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16
    for relu in (False, True):
        got = decode16(_run(tg, kind, A, B, *trans, relu=relu), kind)
        ref = ref_fn(A, B, relu)
        assert_close(got, ref, RTOL, ATOL, f"{kind} {shape} {trans} relu={relu}")
        assert rel_frob(got, ref) <= FROB[kind]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("trans", TRANS)
def test_transposed_many_tiles_per_pair(tg, kind, trans):
    # 16 x 11 = 176 pair tiles of 256 x 256 for 74 CTA pairs: every pair runs
    # two or three tiles, wrapping its TMEM accumulators and ring phases
    # across tiles; ragged in M, N and K
    M, N, K = 4000, 2600, 650
    A, B = synth.normal(M, N, K, seed=2, dtype=kind, scale_by_sqrt_k=True)
    got = decode16(_run(tg, kind, A, B, *trans), kind)
    ref = (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B)
    assert_close(got, ref, RTOL, ATOL, f"{kind} {trans}")
    assert rel_frob(got, ref) <= FROB[kind]


SMALL_M_TB = [(1, 8192, 8192), (3, 1000, 700), (16, 8192, 8192), (17, 520, 333),
              (100, 777, 1200), (128, 14336, 4096), (64, 130, 72)]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("shape", SMALL_M_TB)
def test_small_m_transposed_b(tg, kind, shape):
    # B stored N x K with M <= 128 (the backward product dA = dC . B^T at
    # small batch): the weight-streaming kernel reads K-major weight tiles
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=3, dtype=kind, scale_by_sqrt_k=True)
    ref_fn = oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16
    for relu in (False, True):
        got = decode16(_run(tg, kind, A, B, False, True, relu=relu), kind)
        ref = ref_fn(A, B, relu)
        assert_close(got, ref, RTOL, ATOL, f"{kind} {shape} relu={relu}")
        assert rel_frob(got, ref) <= FROB[kind]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_small_m_transposed_b_bit_exact_and_repeatable(tg, kind):
    M, N, K = 24, 1536, 256
    A, B = synth.integers(M, N, K, seed=1, lo=-1, hi=1, dtype=kind)
    ref = (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B)
    rnd = oracle.round_bf16(ref) if kind == "bf16" else oracle.round_f16(ref)
    assert np.array_equal(decode16(_run(tg, kind, A, B, False, True), kind), decode16(rnd, kind))
    A, B = synth.normal(16, 4096, 8192, seed=3, dtype=kind, scale_by_sqrt_k=True)
    first = _run(tg, kind, A, B, False, True)
    for _ in range(3):
        assert np.array_equal(_run(tg, kind, A, B, False, True), first)


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_transposed_integer_bit_exact(tg, kind):
    M, N, K = 200, 300, 256
    A, B = synth.integers(M, N, K, seed=1, lo=-1, hi=1, dtype=kind)
    ref = (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B)
    rnd = oracle.round_bf16(ref) if kind == "bf16" else oracle.round_f16(ref)
    for trans in TRANS:
        got = _run(tg, kind, A, B, *trans)
        assert np.array_equal(decode16(got, kind), decode16(rnd, kind)), trans


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_matmul_backward(tg, kind):
    import torch
    M, N, K = 384, 264, 520
    A, B = synth.normal(M, N, K, seed=5, dtype=kind, scale_by_sqrt_k=True)
    rng = np.random.default_rng(7)
    G = synth.store(rng.standard_normal((M, N)) * 0.05, kind)
    tdt = torch.bfloat16 if kind == "bf16" else torch.float16
    dA_ = to_dev(A, kind).requires_grad_(True)
    dB_ = to_dev(B, kind).requires_grad_(True)
    C = tg.matmul(dA_, dB_)
    assert C.dtype == tdt and C.shape == (M, N)
    C.backward(to_dev(G, kind))
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    ref_fn = oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16
    # dA = G . B^T and dB = A^T . G with the stored 16-bit values
    ref_dA = ref_fn(G, np.ascontiguousarray(B.T))
    ref_dB = ref_fn(np.ascontiguousarray(A.T), G)
    got_dA = decode16(from_dev(dA_.grad, kind), kind)
    got_dB = decode16(from_dev(dB_.grad, kind), kind)
    assert_close(got_dA, ref_dA, RTOL, ATOL, "dA")
    assert_close(got_dB, ref_dB, RTOL, ATOL, "dB")
    assert rel_frob(got_dA, ref_dA) <= FROB[kind]
    assert rel_frob(got_dB, ref_dB) <= FROB[kind]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("path", ["small_m", "cta_pair"])
@pytest.mark.parametrize("shape", [(128, 14336, 4096), (100, 777, 1200), (3, 1000, 700)])
def test_small_m_transposed_b_follows_tuning_rule(tg, kind, path, shape):
    # A B-transposed call takes the plain call's rule: each forced kernel
    # family gives the oracle's result, ragged shapes included
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=4, dtype=kind, scale_by_sqrt_k=True)
    ref = (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B)
    tg.tune_set([{"op": kind, "path": path, "m_lo": 1, "m_hi": 128}])
    try:
        got = decode16(_run(tg, kind, A, B, False, True), kind)
    finally:
        tg.tune_set([])
    assert_close(got, ref, RTOL, ATOL, f"{kind} {shape} {path}")
    assert rel_frob(got, ref) <= FROB[kind]
