"""GPU parity of the CTA-pair kernel's hybrid schedule against the fp64
oracle, through the C ABI.

When the tiles left for the last wave of the persistent pairs would leave at
least half of the pairs idle, each of those tiles is split into two halves
of its k-blocks; per CTA the first half to finish publishes its fp32 partial
through the workspace and the second adds it into its accumulator before the
ordinary epilogue.  On a 148-SM device (74 pairs) the shapes below have
84 or 96 pair tiles of 256 x 256: 74 whole, 10 or 22 split.  Ragged M, N and K (the
halves then differ in k-block count), every operand layout, ReLU, integer
data bit-exact, and repeated calls bit-identical (the two halves can finish
in either order; a + b gives the same bits as b + a).
"""
import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth
from gpu_util import to_dev, from_dev, decode16, guarded_out, check_guard, assert_close, rel_frob

pytestmark = pytest.mark.gpu
RTOL = ATOL = 1e-2
FROB = {"f16": 2e-3, "bf16": 1e-2}

# 84, 84 and 96 pair tiles: 74 whole, the rest split
SHAPES = [(1792, 3072, 256), (1700, 3000, 130), (1793, 2817, 520)]
TRANS = [(False, False), (True, False), (False, True), (True, True)]


@pytest.fixture(scope="module")
def tg():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_dense_gemm_tma_b200 as tg
    tg.load_library()
    return tg


def _run(tg, kind, A, B, ta=False, tb=False, relu=False):
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


@pytest.mark.parametrize("kind", ["bf16", "f16"])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("trans", TRANS)
def test_split_tail(tg, kind, shape, trans):
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=11, dtype=kind, scale_by_sqrt_k=True)
    ref_fn = oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16
    relu = trans == (True, True)
    bits = _run(tg, kind, A, B, *trans, relu=relu)
    got = decode16(bits, kind)
    ref = ref_fn(A, B, relu)
    assert_close(got, ref, RTOL, ATOL, f"{kind} {shape} {trans}")
    assert rel_frob(got, ref) <= FROB[kind]
    for _ in range(2):
        assert np.array_equal(_run(tg, kind, A, B, *trans, relu=relu), bits), "repeat"


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_split_tail_integer_bit_exact(tg, kind):
    M, N, K = SHAPES[1]
    A, B = synth.integers(M, N, K, seed=12, lo=-2, hi=2, dtype=kind)
    got = _run(tg, kind, A, B)
    ref = (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B)
    rnd = oracle.round_bf16(ref) if kind == "bf16" else oracle.round_f16(ref)
    assert np.array_equal(got, rnd)
