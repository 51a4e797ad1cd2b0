"""Pins of the FP4-weight (WFP4) oracle against what the format and the
mathematics fix, independently of the oracle's own code.

The pages name an FP4-weight GEMM ("TileLang架构深度剖析", test.krestaai.com.au,
performance section) and give no format.  The reading is MXFP4 of the OCP
Microscaling Formats (MX) specification v1.0: E2M1 weight codes, one E8M0
scale 2^(E - 127) per 32 consecutive k of a column, bf16 activations, and
the plain GEMM on the exactly dequantised weight.  Pins:
* every E2M1 code and a set of E8M0 bytes against hand-decoded tables;
* a hand-worked tiny GEMM (golden file);
* exact rational brute force on small shapes, with the element and scale
  values taken from the hand-decoded tables, not from the oracle;
* one-hot activation rows, which must return exactly one dequantised weight
  row (nibble order, block index, scale per column);
* block boundaries with A = ones and a different scale per block;
* the special case of unit scales, which reduces to the bf16 GEMM;
* an independent numpy float64 matmul at a larger size.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _table(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split()
                out[k] = v
    return out


E2M1 = {int(k, 16): Fraction(v) for k, v in _table("e2m1_values.txt").items()}
E8M0 = {int(k): v for k, v in _table("e8m0_values.txt").items()}


def _scale(e):
    """Exact value of an E8M0 byte from the hand-worked table's rule: the
    table lists 2^(E-127) for a few E; other E follow by doubling."""
    if str(e) in ("255",):
        return None
    return Fraction(2) ** (int(e) - 127)


def _bf16_value(bits):
    return Fraction((np.array([bits], np.uint32) << 16).view(np.float32)[0].item())


def test_e2m1_table_has_every_code():
    assert sorted(E2M1) == list(range(16))


def test_golden_e2m1_codes():
    for code, v in E2M1.items():
        got = oracle.e2m1_to_f64(code)
        assert Fraction(got) == v, hex(code)
        if code == 8:
            assert np.signbit(got)              # negative zero


def test_e2m1_structure():
    # sign bit flips the sign; magnitudes rise strictly with codes 0..7
    mags = [E2M1[c] for c in range(8)]
    assert mags == sorted(mags) and len(set(mags)) == 8
    for c in range(8):
        assert E2M1[c | 8] == -E2M1[c]


def test_golden_e8m0_bytes():
    for e, v in E8M0.items():
        got = oracle.e8m0_to_f64(e)
        if v == "nan":
            assert np.isnan(got)
        else:
            assert Fraction(got) == Fraction(v), e
            assert Fraction(v) == _scale(e)      # the table follows 2^(E-127)


def test_golden_wfp4_tiny():
    blocks = {}
    cur = None
    with open(os.path.join(GOLDEN, "wfp4_tiny.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] in ("BQ", "E", "A", "C") and len(parts) == 3:
                cur = parts[0]
                blocks[cur] = []
            else:
                blocks[cur].append(parts)
    Bq = np.array([[int(x, 16) for x in r] for r in blocks["BQ"]], np.uint8)
    E = np.array([[int(x) for x in r] for r in blocks["E"]], np.uint8)
    A = synth.store(np.array(blocks["A"], np.float64), "bf16")
    C = np.array(blocks["C"], np.float64)
    assert np.array_equal(oracle.gemm_wfp4(A, Bq, E, N=3, block=2), C)
    assert np.array_equal(oracle.gemm_wfp4(A, Bq, E, N=3, block=2, relu=True),
                          np.maximum(C, 0.0))


def _exact_w(codes, E, block):
    K, N = codes.shape
    return [[E2M1[int(codes[k, n])] * _scale(E[k // block, n]) for n in range(N)]
            for k in range(K)]


@pytest.mark.parametrize("shape", [(1, 1, 2), (2, 3, 4), (3, 5, 8), (5, 2, 6), (4, 7, 12)])
def test_bruteforce_small_shapes(shape):
    M, N, K = shape
    block = 2
    A, Bq, E, codes = synth.wfp4(M, N, K, seed=11, block=block, e_lo=120, e_hi=134)
    W = _exact_w(codes, E, block)
    C = oracle.gemm_wfp4(A, Bq, E, N=N, block=block)
    for i in range(M):
        a = [_bf16_value(A[i, k]) for k in range(K)]
        for j in range(N):
            exact = sum(a[k] * W[k][j] for k in range(K))
            # a few dyadic products of short significands: the fp64 sum is exact
            assert Fraction(C[i, j]) == exact, (shape, i, j)


def test_one_hot_rows_return_weight_rows():
    K, N = 96, 37                                   # 3 blocks of 32, odd N
    A0, Bq, E, codes = synth.wfp4(1, N, K, seed=5)
    W = _exact_w(codes, E, 32)
    eye = synth.store(np.eye(K), "bf16")
    C = oracle.gemm_wfp4(eye, Bq, E, N=N)
    for k in range(K):
        assert [Fraction(x) for x in C[k]] == W[k], k


def test_block_boundaries():
    K, N = 128, 5
    codes = np.full((K, N), 2, np.uint8)            # every element 1.0
    E = np.array([[127, 128, 126, 130, 120]] * 4, np.uint8)
    E[1] += 1                                       # block 1 doubles, block 3 halves
    E[3] -= 1
    Bq = synth.pack_nibbles(codes)
    ones = synth.store(np.ones((1, K)), "bf16")
    C = oracle.gemm_wfp4(ones, Bq, E, N=N)
    for n in range(N):
        expect = sum(32 * _scale(E[b, n]) for b in range(4))
        assert Fraction(C[0, n]) == expect


def test_unit_scales_reduce_to_bf16_gemm():
    M, N, K = 9, 40, 64
    A, Bq, _, codes = synth.wfp4(M, N, K, seed=3)
    E = np.full((K // 32, N), 127, np.uint8)
    W = oracle.dequant_fp4(Bq, E, N)
    # every E2M1 value is exact in bf16, so W's bf16 bit patterns hold W
    W_bits = oracle.round_bf16(W)
    assert np.array_equal(oracle.bf16_to_f64(W_bits), W)
    assert np.array_equal(oracle.gemm_wfp4(A, Bq, E, N=N), oracle.gemm_bf16(A, W_bits))


def test_numpy_float64_crosscheck():
    M, N, K = 64, 96, 256
    A, Bq, E, codes = synth.wfp4(M, N, K, seed=8)
    W = np.array([[float(v) for v in row] for row in _exact_w(codes, E, 32)])
    Ad = oracle.bf16_to_f64(A)
    ref = np.matmul(Ad, W)
    C = oracle.gemm_wfp4(A, Bq, E, N=N)
    assert np.max(np.abs(C - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_nan_scale_poisons_its_column():
    K, N = 64, 4
    A, Bq, E, _ = synth.wfp4(2, N, K, seed=2)
    E = E.copy()
    E[1, 2] = 255
    C = oracle.gemm_wfp4(A, Bq, E, N=N)
    assert np.all(np.isnan(C[:, 2]))
    assert not np.any(np.isnan(C[:, [0, 1, 3]]))
