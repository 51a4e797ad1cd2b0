"""GPU parity of the operand-swapped CTA-pair kernel against the fp64 oracle.

A 16-bit GEMM with M <= 128 on the CTA-pair path runs with its operands
swapped: the kernel computes C^T = B^T . A^T with 128-column pair tiles (the
weight columns on its 256-row side, the M activation rows on its
128-column side) and writes the tile transposed into C.  That is the default
for 64 < M <= 128 and N >= 4096; a tuning rule forces it for other shapes.

Shapes: ragged M (a partial 64-row store), ragged N (not a multiple of the
256-column pair tile or of a 32-column store), ragged K, ReLU, B stored
K x N and N x K, both dtypes, integer data bit-exact, few pair tiles (the
last wave split along K, partials through the workspace), repeatability,
and the full-size 128 x 14336 x 4096 on sampled columns.
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


def _run(tg, kind, A, B, tb=False, relu=False, force=True):
    import torch
    M, K = A.shape
    N = B.shape[1]
    big, C, pad = guarded_out(M, N, kind)
    fn = tg.gemm_bf16 if kind == "bf16" else tg.gemm_f16
    Bs = np.ascontiguousarray(B.T) if tb else B
    if force:
        tg.tune_set([{"op": kind, "path": "cta_pair", "m_lo": 1, "m_hi": 128}])
    try:
        fn(to_dev(A, kind), to_dev(Bs, kind), C=C, relu=relu, trans_b=tb)
        torch.cuda.synchronize()
    finally:
        if force:
            tg.tune_set([])
    assert tg.last_device_status() == 0
    check_guard(big, kind, M, N, pad)
    return from_dev(C, kind)


def _ref(kind, A, B, relu=False):
    return (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B, relu)


SHAPES = [(65, 4104, 1000), (100, 520, 200), (128, 8192, 640), (1, 300, 64), (17, 2000, 1024),
          (128, 256, 4096), (127, 1000, 72)]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("tb", [False, True])
def test_swapped_pair(tg, kind, shape, tb):
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=6, dtype=kind, scale_by_sqrt_k=True)
    for relu in (False, True):
        got = decode16(_run(tg, kind, A, B, tb, relu), kind)
        ref = _ref(kind, A, B, relu)
        assert_close(got, ref, RTOL, ATOL, f"{kind} {shape} tb={tb} relu={relu}")
        assert rel_frob(got, ref) <= FROB[kind]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("shape", [(128, 2048, 1024), (96, 3000, 4096)])
def test_swapped_pair_split_last_wave(tg, kind, shape):
    # 8 and 12 pair tiles for 74 CTA pairs: each tile is split into two
    # halves of its k-blocks that meet through the workspace
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=7, dtype=kind, scale_by_sqrt_k=True)
    got = decode16(_run(tg, kind, A, B), kind)
    ref = _ref(kind, A, B)
    assert_close(got, ref, RTOL, ATOL, f"{kind} {shape}")
    assert rel_frob(got, ref) <= FROB[kind]


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_swapped_pair_bit_exact_and_repeatable(tg, kind):
    M, N, K = 96, 1000, 256
    A, B = synth.integers(M, N, K, seed=1, lo=-1, hi=1, dtype=kind)
    ref = _ref(kind, A, B)
    rnd = oracle.round_bf16(ref) if kind == "bf16" else oracle.round_f16(ref)
    for tb in (False, True):
        assert np.array_equal(decode16(_run(tg, kind, A, B, tb), kind), decode16(rnd, kind))
    A, B = synth.normal(128, 4096, 4096, seed=3, dtype=kind, scale_by_sqrt_k=True)
    first = _run(tg, kind, A, B)
    for _ in range(3):
        assert np.array_equal(_run(tg, kind, A, B), first)


def test_swapped_pair_full_size_sampled(tg):
    # the 128 x 14336 x 4096 workload on its default path, B stored both ways;
    # 256 sampled columns against the oracle
    M, N, K = 128, 14336, 4096
    A, B = synth.normal(M, N, K, seed=3, dtype="bf16", scale_by_sqrt_k=True)
    cols = np.arange(9000, 9256)
    ref = oracle.gemm_bf16(A, np.ascontiguousarray(B[:, cols]))
    for tb in (False, True):
        got = decode16(_run(tg, "bf16", A, B, tb, force=False), "bf16")
        assert_close(got[:, cols], ref, RTOL, ATOL, f"tb={tb}")
        assert rel_frob(got[:, cols], ref) <= FROB["bf16"]
