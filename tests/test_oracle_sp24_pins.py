"""Pins of the oracle's 2:4 structured-sparse GEMM (oracle.gemm_sp24 and
oracle.expand_sp24) against facts fixed independently of its code:

* a hand-worked example (tests/golden/sp24_tiny.txt) whose codes were decoded
  by hand, with B rows that no kept value may touch;
* one-hot compressed values: each kept value lands on exactly the dense k its
  code names, for every one of the 16 codes in both nibbles of a byte;
* the generator's own record of each kept value's k (drawn as integer pairs,
  not decoded from the bytes) builds the dense A, and numpy's float64 matmul
  of it must agree;
* exact rational brute force on tiny integer inputs;
* the all-(0, 1) code reduces to the dense GEMM of a matrix with two leading
  non-zeros per chunk, checked against the pinned dense oracle.
"""
import itertools
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read_golden():
    blocks, cur = {}, None
    with open(os.path.join(GOLDEN, "sp24_tiny.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] in ("AC", "E", "B", "C") and len(parts) == 3:
                cur = parts[0]
                blocks[cur] = []
            else:
                blocks[cur].append(parts)
    return blocks


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_golden_sp24_tiny(dtype):
    g = _read_golden()
    Ac = synth.store(np.array([[float(x) for x in r] for r in g["AC"]]), dtype)
    E = np.array([[int(x, 16) for x in r] for r in g["E"]], np.uint8)
    B = synth.store(np.array([[float(x) for x in r] for r in g["B"]]), dtype)
    C = np.array([[float(x) for x in r] for r in g["C"]])
    assert np.array_equal(oracle.gemm_sp24(Ac, E, B, dtype), C)
    dense = oracle.expand_sp24(Ac, E, 8, dtype)
    assert np.array_equal(dense[0], [0, 2, 0, -1, 0.5, 0, 4, 0])
    assert np.array_equal(dense[1], [3, 1, 0, 0, 0, 0, -2, 1])
    # ReLU after the sum
    Bn = synth.store(-np.array([[float(x) for x in r] for r in g["B"]]), dtype)
    assert np.array_equal(oracle.gemm_sp24(Ac, E, Bn, dtype, relu=True), np.zeros((2, 2)))


@pytest.mark.parametrize("chunk", [0, 1])
def test_one_hot_values_land_on_the_coded_position(chunk):
    # K = 8: two chunks share one byte; every code in either nibble
    for code in range(16):
        for p in (0, 1):
            Ac = np.zeros((1, 4), np.float64)
            Ac[0, 2 * chunk + p] = 1.0
            byte = code << 4 if chunk else code
            E = np.array([[byte]], np.uint8)
            dense = oracle.expand_sp24(synth.store(Ac, "bf16"), E, 8, "bf16")
            idx = (code >> (2 * p)) & 3            # bits 0-1 for the first value, 2-3 the second
            want = np.zeros(8)
            want[4 * chunk + idx] = 1.0
            assert np.array_equal(dense[0], want), (chunk, code, p)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_generator_positions_and_numpy(dtype):
    M, N, K = 37, 29, 96
    Ac, E, B, pos = synth.sp24(M, N, K, seed=11, dtype=dtype)
    dec = oracle.bf16_to_f64 if dtype == "bf16" else oracle.f16_to_f64
    vals = dec(Ac)
    A = np.zeros((M, K))
    A[np.arange(M)[:, None], pos] = vals          # the generator's k of each kept value
    assert np.array_equal(oracle.expand_sp24(Ac, E, K, dtype), A)
    ref = A @ dec(B)
    got = oracle.gemm_sp24(Ac, E, B, dtype)
    assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
    # every chunk keeps two distinct positions, all six pairs occur
    pairs = pos.reshape(M, K // 4, 2) - 4 * np.arange(K // 4)[None, :, None]
    assert np.all(pairs[..., 0] < pairs[..., 1])
    assert len({tuple(p) for p in pairs.reshape(-1, 2)}) == 6


def test_exact_brute_force_tiny():
    for M, N, K in itertools.product((1, 2, 3), (1, 2, 3), (4, 8)):
        Ac, E, B, pos = synth.sp24(M, N, K, seed=M * 100 + N * 10 + K, dtype="bf16", a_int=3)
        a = oracle.bf16_to_f64(Ac)
        b = oracle.bf16_to_f64(B)
        got = oracle.gemm_sp24(Ac, E, B, "bf16")
        for i in range(M):
            for j in range(N):
                exact = sum(Fraction(a[i, t]) * Fraction(b[pos[i, t], j]) for t in range(K // 2))
                assert Fraction(got[i, j]) == exact


def test_leading_pair_code_is_the_dense_gemm():
    M, N, K = 20, 24, 64
    rng = np.random.default_rng(3)
    vals = synth.store(rng.standard_normal((M, K // 2)), "bf16")
    E = np.full((M, K // 8), 0x44, np.uint8)          # code 4 = (0, 1) in both nibbles
    B = synth.store(rng.standard_normal((K, N)), "bf16")
    dense = np.zeros((M, K), np.uint16)
    dense[:, 0::4] = vals[:, 0::2]
    dense[:, 1::4] = vals[:, 1::2]
    assert np.array_equal(oracle.gemm_sp24(vals, E, B, "bf16"), oracle.gemm_bf16(dense, B))
