"""GPU parity of the 2:4 structured-sparse GEMM (tg_gemm_sp24_f16 / _bf16:
compressed A values plus 2-bit position codes, dense B, sparse tensor-core
MMAs) against the fp64 oracle, which expands A and runs the plain GEMM.

Tolerance as for the dense 16-bit GEMM: rtol = atol = 1e-2 elementwise,
relative Frobenius error <= 2e-3 (fp16) / 1e-2 (bf16).  Integer-valued
inputs give exact fp32 sums, so the one rounding to the output type must
match the oracle's bit for bit.  Every random case draws all six position
pairs in every code slot; shapes cover ragged M, N and K (K not a multiple
of the 64 dense k a stage holds, nor of the 128 a code block holds), one
tile, and more tiles than CTAs.  A wrong reading of the codes' layout in
tensor memory moves values onto the wrong rows of B and fails at once.
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


def _run(tg, kind, Ac, E, B, relu=False, guard=True):
    import torch
    M, N = Ac.shape[0], B.shape[1]
    C = None
    if guard:
        big, C, pad = guarded_out(M, N, kind)
    C = tg.gemm_sp24(to_dev(Ac, kind), to_dev(E, "u8"), to_dev(B, kind), C=C, relu=relu)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    if guard:
        check_guard(big, kind, M, N, pad)
    return from_dev(C, kind)


SHAPES = [(128, 256, 64), (1, 24, 32), (300, 520, 200), (129, 257, 1000), (640, 264, 4096),
          (2048, 2560, 256)]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("relu", [False, True])
def test_random(tg, kind, shape, relu):
    M, N, K = shape
    Ac, E, B, _ = synth.sp24(M, N, K, seed=2, dtype=kind)
    got = decode16(_run(tg, kind, Ac, E, B, relu), kind)
    ref = oracle.gemm_sp24(Ac, E, B, kind, relu)
    assert_close(got, ref, RTOL, ATOL, f"{kind} {shape} relu={relu}")
    assert rel_frob(got, ref) <= FROB[kind]
    if relu:
        assert np.all(got >= 0)


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_integer_bit_exact(tg, kind):
    for M, N, K in ((200, 300, 256), (64, 256, 2048)):
        Ac, E, B, _ = synth.sp24(M, N, K, seed=1, dtype=kind, a_int=2)
        ref = oracle.gemm_sp24(Ac, E, B, kind)
        rnd = oracle.round_bf16(ref) if kind == "bf16" else oracle.round_f16(ref)
        assert np.array_equal(decode16(_run(tg, kind, Ac, E, B), kind), decode16(rnd, kind))


def test_each_position_pair_alone(tg):
    # every chunk of the matrix uses the same pair: each of the six in turn
    M, N, K = 256, 256, 512
    rng = np.random.default_rng(5)
    Ac = synth.store(rng.integers(-3, 4, size=(M, K // 2)).astype(np.float64), "bf16")
    B = synth.store(rng.integers(-3, 4, size=(K, N)).astype(np.float64), "bf16")
    for i0, i1 in synth.SP24_PAIRS:
        code = i0 | (i1 << 2)
        E = np.full((M, K // 8), code | (code << 4), np.uint8)
        ref = oracle.gemm_sp24(Ac, E, B, "bf16")
        got = _run(tg, "bf16", Ac, E, B)
        assert np.array_equal(decode16(got, "bf16"), decode16(oracle.round_bf16(ref), "bf16")), (i0, i1)


@pytest.mark.parametrize("size", [4096, 8192])
def test_full_size_sampled(tg, size):
    M = N = K = size
    Ac, E, B, _ = synth.sp24(M, N, K, seed=2, dtype="bf16")
    got = decode16(_run(tg, "bf16", Ac, E, B, guard=False), "bf16")
    rng = np.random.default_rng(17)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 40, replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 40, replace=False)]))
    ref_r = oracle.gemm_sp24(np.ascontiguousarray(Ac[rows]), np.ascontiguousarray(E[rows]), B, "bf16")
    ref_c = oracle.gemm_sp24(Ac, E, np.ascontiguousarray(B[:, cols]), "bf16")
    assert_close(got[rows], ref_r, RTOL, ATOL, "rows")
    assert_close(got[:, cols], ref_c, RTOL, ATOL, "cols")
    assert rel_frob(got[rows], ref_r) <= FROB["bf16"]
    assert rel_frob(got[:, cols], ref_c) <= FROB["bf16"]


def test_repeatable(tg):
    Ac, E, B, _ = synth.sp24(1024, 2048, 2048, seed=3, dtype="f16")
    first = _run(tg, "f16", Ac, E, B, guard=False)
    for _ in range(3):
        assert np.array_equal(_run(tg, "f16", Ac, E, B, guard=False), first)
