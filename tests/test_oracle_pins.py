"""Pins for the CPU oracle: it is checked against things other than itself.

* hand-worked fixtures in tests/golden/ (integer GEMM, 4-bit decoding, a
  dequantize GEMM, output rounding);
* exact rational brute force (fractions.Fraction) on every tiny shape;
* closed forms: all-ones, identity, permutation, rank-one;
* an independent library routine (numpy float64 matmul);
* exhaustive decoding of every fp16 / bf16 bit pattern against numpy;
* round-to-nearest-even against numpy's float16 cast and against a
  brute-force nearest-value search over every finite bf16 value.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------- helpers

def _read_blocks(name):
    """Parse a golden file of '<TAG> rows cols' headers followed by rows."""
    blocks, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0].isalpha() and parts[0].isupper() and len(parts) == 3:
                cur = parts[0]
                blocks[cur] = []
            else:
                blocks[cur].append(parts)
    return blocks


def _np_f16_decode(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def _np_bf16_decode(bits):
    u = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):         # signalling-NaN patterns are expected here
        return u.view(np.float32).astype(np.float64)


def _exact(Ad, Bd):
    """Exact rational product of two float64-valued matrices."""
    M, K = Ad.shape
    N = Bd.shape[1]
    return [[sum((Fraction(float(Ad[i, k])) * Fraction(float(Bd[k, j])) for k in range(K)),
                 Fraction(0)) for j in range(N)] for i in range(M)]


def _check_against_exact(C, Ad, Bd):
    """|C - exact| <= K * 2^-52 * sum|a||b| elementwise (fp64 summation bound)."""
    E = _exact(Ad, Bd)
    K = Ad.shape[1]
    bound = np.abs(Ad) @ np.abs(Bd) * (K * 2.0 ** -52) + 1e-300
    for i in range(C.shape[0]):
        for j in range(C.shape[1]):
            err = abs(Fraction(float(C[i, j])) - E[i][j])
            assert err <= Fraction(float(bound[i, j])), (i, j, float(err))


# ------------------------------------------------------------- golden fixtures

def test_golden_integer_gemm():
    b = _read_blocks("gemm_int_2x3x2.txt")
    A = np.array(b["A"], np.float32)
    B = np.array(b["B"], np.float32)
    C = np.array(b["C"], np.float64)
    assert np.array_equal(oracle.gemm_f32(A, B), C)
    A2 = A.copy()
    A2[1] *= -1
    C2 = C.copy()
    C2[1] = 0.0
    assert np.array_equal(oracle.gemm_f32(A2, B, relu=True), C2)
    # the same through the 16-bit decoders (all values exact in fp16 / bf16)
    assert np.array_equal(oracle.gemm_f16(synth.store(A, "f16"), synth.store(B, "f16")), C)
    assert np.array_equal(oracle.gemm_bf16(synth.store(A, "bf16"), synth.store(B, "bf16")), C)


def test_golden_nibbles():
    data = []
    with open(os.path.join(GOLDEN, "int4_nibbles.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                h, lo, hi = line.split()
                data.append((int(h, 16), int(lo), int(hi)))
    assert len(data) >= 10
    Bq = np.array([[d[0] for d in data]], np.uint8)          # 1 x n bytes
    N = 2 * Bq.shape[1]
    one = synth.store(np.ones((1, N)), "f16")                # scale 1.0
    W = oracle.dequant_w4(Bq, one, N, group=1)
    expect = np.array([[v for d in data for v in (d[1], d[2])]], np.float64)
    assert np.array_equal(W, expect)


def test_golden_w4a16_tiny():
    b = _read_blocks("w4a16_tiny.txt")
    Bq = np.array([[int(x, 16) for x in r] for r in b["BQ"]], np.uint8)
    S = synth.store(np.array(b["S"], np.float64), "f16")
    A = synth.store(np.array(b["A"], np.float64), "f16")
    C = np.array(b["C"], np.float64)
    out = oracle.gemm_w4a16(A, Bq, S, N=3, group=2)
    assert np.array_equal(out, C)


def test_golden_rounding():
    with open(os.path.join(GOLDEN, "rounding.txt")) as f:
        n = 0
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            kind, expr, hexbits = line.split()
            x = float(eval(expr, {"__builtins__": {}}))
            fn = oracle.round_f16 if kind == "f16" else oracle.round_bf16
            got = int(fn(np.array([x]))[0])
            assert got == int(hexbits, 16), (kind, expr, hex(got))
            n += 1
    assert n >= 20


# ------------------------------------------------------------- brute force

TINY = list(itertools.product(range(1, 6), repeat=3)) + [(7, 9, 13)]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_bruteforce_tiny_shapes(dtype):
    rng = np.random.default_rng(123)
    fn = {"f32": oracle.gemm_f32, "f16": oracle.gemm_f16, "bf16": oracle.gemm_bf16}[dtype]
    dec = {"f32": lambda a: a.astype(np.float64), "f16": _np_f16_decode,
           "bf16": _np_bf16_decode}[dtype]
    for (M, N, K) in TINY:
        A = synth.store(rng.uniform(-1, 1, (M, K)), dtype)
        B = synth.store(rng.uniform(-1, 1, (K, N)), dtype)
        C = fn(A, B)
        _check_against_exact(C, dec(A), dec(B))
        Cr = fn(A, B, relu=True)
        assert np.array_equal(Cr, np.maximum(C, 0.0))


def test_bruteforce_w4a16_tiny():
    rng = np.random.default_rng(7)
    for (M, N, K) in [(1, 1, 4), (2, 3, 4), (3, 5, 8), (4, 7, 6), (5, 2, 10)]:
        A = synth.store(rng.uniform(-1, 1, (M, K)), "f16")
        q = rng.integers(-8, 8, (K, N))
        Bq = synth.pack_int4(q)
        s = synth.store(rng.uniform(0.005, 0.02, ((K + 1) // 2, N)), "f16")
        Wd = q.astype(np.float64) * np.repeat(_np_f16_decode(s), 2, axis=0)[:K]
        C = oracle.gemm_w4a16(A, Bq, s, N=N, group=2)
        _check_against_exact(C, _np_f16_decode(A), Wd)


# ------------------------------------------------------------- closed forms

def test_all_ones_gives_k():
    for (M, N, K) in [(3, 5, 1), (17, 9, 300), (64, 33, 4096)]:
        A = np.ones((M, K), np.float32)
        B = np.ones((K, N), np.float32)
        assert np.all(oracle.gemm_f32(A, B) == K)
        A16 = synth.store(np.ones((M, K)), "bf16")
        B16 = synth.store(np.ones((K, N)), "bf16")
        assert np.all(oracle.gemm_bf16(A16, B16) == K)


def test_identity_and_permutation():
    rng = np.random.default_rng(5)
    n, N = 37, 23
    B = rng.standard_normal((n, N)).astype(np.float32)
    I = np.eye(n, dtype=np.float32)
    assert np.array_equal(oracle.gemm_f32(I, B), B.astype(np.float64))
    perm = rng.permutation(n)
    P = I[perm]
    assert np.array_equal(oracle.gemm_f32(P, B), B[perm].astype(np.float64))
    # identity on the right returns A
    A = rng.standard_normal((11, n)).astype(np.float32)
    assert np.array_equal(oracle.gemm_f32(A, I), A.astype(np.float64))
    Bh = synth.store(B, "f16")
    assert np.array_equal(oracle.gemm_f16(synth.store(P, "f16"), Bh), _np_f16_decode(Bh)[perm])


def test_rank_one():
    # A = u 1^T, B = 1 v^T  ->  C = K u v^T  (powers of two keep it exact)
    M, N, K = 9, 14, 64
    u = 2.0 ** np.arange(-4, M - 4)
    v = -(2.0 ** np.arange(-7, N - 7))
    A = np.repeat(u[:, None], K, axis=1).astype(np.float32)
    B = np.repeat(v[None, :], K, axis=0).astype(np.float32)
    assert np.array_equal(oracle.gemm_f32(A, B), K * np.outer(u, v))


def test_integer_exact_against_int64():
    rng = np.random.default_rng(11)
    M, N, K = 64, 48, 300
    Ai = rng.integers(-3, 4, (M, K))
    Bi = rng.integers(-3, 4, (K, N))
    ref = (Ai @ Bi).astype(np.float64)
    assert np.array_equal(oracle.gemm_f32(Ai.astype(np.float32), Bi.astype(np.float32)), ref)
    assert np.array_equal(oracle.gemm_bf16(synth.store(Ai, "bf16"), synth.store(Bi, "bf16")), ref)


def test_numpy_float64_crosscheck():
    for (M, N, K), seed in [((256, 256, 256), 0), ((64, 96, 200), 1)]:
        A, B = synth.uniform_pm1(M, N, K, seed)
        C = oracle.gemm_f32(A, B)
        ref = A.astype(np.float64) @ B.astype(np.float64)
        scale = np.abs(A.astype(np.float64)) @ np.abs(B.astype(np.float64))
        assert np.max(np.abs(C - ref) / scale) <= 1e-12
        # a transposed operand would fail: check non-square shape really is (M, N)
        assert C.shape == (M, N)


def test_relu_flag():
    A, B = synth.normal(40, 50, 60, 3)
    C = oracle.gemm_f32(A, B)
    Cr = oracle.gemm_f32(A, B, relu=True)
    assert np.array_equal(Cr, np.where(C < 0, 0.0, C))
    assert np.count_nonzero(Cr == 0) == np.count_nonzero(C <= 0)
    assert 0 < np.count_nonzero(C < 0) < C.size


# ------------------------------------------------------------- decoders

def test_f16_decode_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.f16_to_f64(bits)
    ref = _np_f16_decode(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_decode_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_f64(bits)
    ref = _np_bf16_decode(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ------------------------------------------------------------- rounding

def _rounding_probe(rng, lo_exp, hi_exp, n):
    mant = rng.uniform(1.0, 2.0, n)
    ex = rng.integers(lo_exp, hi_exp, n)
    x = np.ldexp(mant, ex) * rng.choice([-1.0, 1.0], n)
    return x


def test_round_f16_matches_numpy():
    rng = np.random.default_rng(9)
    x = _rounding_probe(rng, -27, 17, 200000)
    # exact ties and near-ties: midpoints between adjacent fp16 values
    bits = rng.integers(0, 0x7BFF, 20000).astype(np.uint16)
    a = _np_f16_decode(bits)
    b = _np_f16_decode(bits + 1)
    mids = (a + b) / 2
    x = np.concatenate([x, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9)])
    got = oracle.round_f16(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def test_round_bf16_nearest_even_bruteforce():
    # every finite non-negative bf16 value, in increasing order
    pos = np.arange(0, 0x7F80, dtype=np.uint32).astype(np.uint16)
    vals = _np_bf16_decode(pos)
    rng = np.random.default_rng(10)
    x = np.abs(_rounding_probe(rng, -135, 127, 100000))
    mids = (vals[:-1] + vals[1:]) / 2
    pick = rng.integers(0, len(mids), 20000)
    x = np.concatenate([x, mids[pick], np.nextafter(mids[pick], 0), np.nextafter(mids[pick], np.inf)])
    idx = np.searchsorted(vals, x)                    # vals[idx-1] < x <= vals[idx]
    idx = np.clip(idx, 1, len(vals) - 1)
    lo, hi = vals[idx - 1], vals[idx]
    dlo, dhi = x - lo, hi - x
    choose_hi = (dhi < dlo) | ((dhi == dlo) & ((pos[idx] & 1) == 0))
    exact = vals[idx] == x
    ref = np.where(exact | choose_hi, pos[idx], pos[idx - 1]).astype(np.uint16)
    got = oracle.round_bf16(x)
    assert np.array_equal(got, ref)
    # the sign is carried through
    assert np.array_equal(oracle.round_bf16(-x), ref | 0x8000)


# ------------------------------------------------------------- 4-bit weights

def test_w4_one_hot_rows_pick_dequantised_rows():
    rng = np.random.default_rng(4)
    K, N = 256, 10
    q = rng.integers(-8, 8, (K, N))
    q[0, :2] = [-8, 7]                     # extremes of the signed range
    Bq = synth.pack_int4(q)
    s = synth.store(rng.uniform(0.005, 0.02, (K // 128, N)), "f16")
    sd = _np_f16_decode(s)
    for k in [0, 1, 127, 128, 255]:
        a = np.zeros((1, K))
        a[0, k] = 1.0
        C = oracle.gemm_w4a16(synth.store(a, "f16"), Bq, s, N=N)
        assert np.array_equal(C[0], q[k] * sd[k // 128]), k


def test_w4_group_boundaries_with_ones():
    rng = np.random.default_rng(6)
    K, N = 512, 6
    q = rng.integers(-8, 8, (K, N))
    s_vals = np.array([[2.0 ** -6], [2.0 ** -5], [2.0 ** -4], [2.0 ** -3]]) * np.ones((1, N))
    s = synth.store(s_vals, "f16")
    C = oracle.gemm_w4a16(synth.store(np.ones((1, K)), "f16"), synth.pack_int4(q), s, N=N)
    expect = sum(s_vals[g] * q[128 * g:128 * (g + 1)].sum(axis=0) for g in range(4))
    assert np.array_equal(C[0], expect)


def test_w4_dequant_matches_generator_q():
    A, Bq, s, q = synth.w4a16(3, 37, 256, seed=4)
    W = oracle.dequant_w4(Bq, s, 37)
    assert np.array_equal(W, q.astype(np.float64) * np.repeat(_np_f16_decode(s), 128, axis=0))


def test_oracle_error_bound_is_far_below_tolerances():
    # fp64 summation error bound K * 2^-53 relative to sum|a||b|, at the
    # largest K used (8192), is < 1e-12: 10^7 below the tightest tolerance.
    assert 8192 * 2.0 ** -53 < 1e-12
    assert math.isclose(2.0 ** -53, 1.1102230246251565e-16)
