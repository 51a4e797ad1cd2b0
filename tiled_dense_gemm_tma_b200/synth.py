"""Seeded synthetic inputs for the GEMM paths.

This module draws and stores input matrices; it holds none of the GEMM's
arithmetic and imports neither the CUDA binding nor the oracle, so both
sides of a parity test can take their inputs from here.

Recipe (the pages fix no input data; the distributions are those of the
library's benchmark workloads):

* ``numpy.random.default_rng(seed)`` (PCG64) is the only source.  Draws are
  made in the order A, then B (then q, then scales for the 4-bit path), each
  matrix row-major in one call.
* Real values are drawn in float64 and rounded once to the storage type:
  float32 and float16 by numpy's round-to-nearest-even casts; bfloat16 by
  rounding to float32 first and then to bfloat16 with round-to-nearest-even
  on the bit pattern (so bf16 values are double-rounded through fp32; any
  deterministic rounding serves, since both sides read the stored values).
* fp16 / bf16 matrices are returned as uint16 bit-pattern arrays.
* The 4-bit weight q (integers in [-8, 7]) is packed two per byte, column
  2j in the low nibble and 2j+1 in the high nibble of byte j of its row.
  FP4 (E2M1) weight codes 0..15 are packed the same way; their E8M0 scale
  exponents are stored one byte each.
"""
import math

import numpy as np


def _to_bf16_bits(x64):
    f32 = np.asarray(x64, np.float64).astype(np.float32)
    u = f32.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(f32)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def _to_f16_bits(x64):
    return np.asarray(x64, np.float64).astype(np.float16).view(np.uint16)


def store(x64, dtype):
    """Round float64 draws to a storage type: 'f32', 'f16' or 'bf16'."""
    if dtype == "f32":
        return np.asarray(x64, np.float64).astype(np.float32)
    if dtype == "f16":
        return _to_f16_bits(x64)
    if dtype == "bf16":
        return _to_bf16_bits(x64)
    raise ValueError(dtype)


def pack_nibbles(codes):
    """Pack 4-bit codes (K x N, values 0..15) into K x ceil(N/2) bytes:
    column 2j in the low nibble and 2j+1 in the high nibble of byte j."""
    c = np.asarray(codes)
    if c.min(initial=0) < 0 or c.max(initial=0) > 15:
        raise ValueError("code out of [0, 15]")
    K, N = c.shape
    nib = c.astype(np.uint8)
    if N % 2:
        nib = np.concatenate([nib, np.zeros((K, 1), np.uint8)], axis=1)
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def pack_int4(q):
    """Pack an int array (K x N, values in [-8, 7]) into K x ceil(N/2) bytes
    (two's complement nibbles, as pack_nibbles)."""
    q = np.asarray(q)
    if q.min(initial=0) < -8 or q.max(initial=0) > 7:
        raise ValueError("q out of [-8, 7]")
    return pack_nibbles(q.astype(np.int64) & 0xF)


def uniform_pm1(M, N, K, seed, dtype="f32"):
    """A (M x K), B (K x N) with i.i.d. uniform[-1, 1] entries."""
    rng = np.random.default_rng(seed)
    A = rng.uniform(-1.0, 1.0, size=(M, K))
    B = rng.uniform(-1.0, 1.0, size=(K, N))
    return store(A, dtype), store(B, dtype)


def normal(M, N, K, seed, dtype="f32", scale_by_sqrt_k=False):
    """A, B with i.i.d. N(0, 1) entries, optionally divided by sqrt(K)."""
    rng = np.random.default_rng(seed)
    s = 1.0 / math.sqrt(K) if (scale_by_sqrt_k and K > 0) else 1.0
    A = rng.standard_normal(size=(M, K)) * s
    B = rng.standard_normal(size=(K, N)) * s
    return store(A, dtype), store(B, dtype)


def integers(M, N, K, seed, lo=-3, hi=3, dtype="f32"):
    """A, B with i.i.d. integer entries uniform in {lo..hi}."""
    rng = np.random.default_rng(seed)
    A = rng.integers(lo, hi + 1, size=(M, K)).astype(np.float64)
    B = rng.integers(lo, hi + 1, size=(K, N)).astype(np.float64)
    return store(A, dtype), store(B, dtype)


def w4a16(M, N, K, seed, group=128, s_lo=0.005, s_hi=0.02, a_int=None):
    """Inputs of the 4-bit-weight GEMM.

    Returns (A fp16 bits M x K, Bq packed uint8 K x ceil(N/2), scales fp16
    bits ceil(K/group) x N, q int8 K x N).  A is N(0, 1), or integers in
    [-a_int, a_int] when a_int is given; q is uniform in {-8..7}; scales are
    uniform[s_lo, s_hi] rounded to fp16.
    """
    rng = np.random.default_rng(seed)
    if a_int is None:
        A = rng.standard_normal(size=(M, K))
    else:
        A = rng.integers(-a_int, a_int + 1, size=(M, K)).astype(np.float64)
    q = rng.integers(-8, 8, size=(K, N)).astype(np.int8)
    G = (K + group - 1) // group
    s = rng.uniform(s_lo, s_hi, size=(G, N))
    return store(A, "f16"), pack_int4(q), store(s, "f16"), q


def wfp4(M, N, K, seed, block=32, e_lo=118, e_hi=122, a_int=None):
    """Inputs of the FP4-weight GEMM (MXFP4 weights, bf16 activations).

    Returns (A bf16 bits M x K, Bq packed uint8 K x ceil(N/2) of E2M1 codes,
    scales uint8 E8M0 exponents ceil(K/block) x N, codes uint8 K x N).  A is
    N(0, 1), or integers in [-a_int, a_int] when a_int is given; the codes
    are uniform over all 16 E2M1 codes; the scale exponents are uniform in
    {e_lo..e_hi} (2^-9 .. 2^-5 by default).
    """
    rng = np.random.default_rng(seed)
    if a_int is None:
        A = rng.standard_normal(size=(M, K))
    else:
        A = rng.integers(-a_int, a_int + 1, size=(M, K)).astype(np.float64)
    codes = rng.integers(0, 16, size=(K, N)).astype(np.uint8)
    G = (K + block - 1) // block
    E = rng.integers(e_lo, e_hi + 1, size=(G, N)).astype(np.uint8)
    return store(A, "bf16"), pack_nibbles(codes), E, codes


def with_ld(X, ld):
    """Copy a 2-D array into a wider row pitch ld (extra columns zero)."""
    R, C = X.shape
    if ld < C:
        raise ValueError("ld < columns")
    out = np.zeros((R, ld), X.dtype)
    out[:, :C] = X
    return out[:, :C]


# The six increasing position pairs (i0 < i1) a chunk of 4 can keep.
SP24_PAIRS = ((0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3))


def sp24(M, N, K, seed, dtype="bf16", scale_by_sqrt_k=True, a_int=None):
    """Inputs of the 2:4 structured-sparse GEMM (sparse A, dense B).

    Each chunk of 4 consecutive k of a row of A keeps two positions, a pair
    drawn uniformly from the six increasing pairs.  Returns (Ac 16-bit bits
    M x K/2: the kept values in increasing k; E uint8 M x ceil(K/8): position
    codes, i0 | i1 << 2 per chunk, even chunk in the low nibble; B bits
    K x N; pos int M x K/2: the k of each kept value).  Kept values are
    N(0, 1) / sqrt(K / 2) (or integers in [-a_int, a_int]); B is
    N(0, 1) / sqrt(K).  K must be a multiple of 4.
    """
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    rng = np.random.default_rng(seed)
    C4 = K // 4
    which = rng.integers(0, 6, size=(M, C4))
    if a_int is None:
        s = 1.0 / math.sqrt(max(K // 2, 1)) if scale_by_sqrt_k else 1.0
        vals = rng.standard_normal(size=(M, K // 2)) * s
    else:
        vals = rng.integers(-a_int, a_int + 1, size=(M, K // 2)).astype(np.float64)
    sb = 1.0 / math.sqrt(K) if (scale_by_sqrt_k and K > 0) else 1.0
    B = rng.standard_normal(size=(K, N)) * sb if a_int is None else \
        rng.integers(-a_int, a_int + 1, size=(K, N)).astype(np.float64)
    pairs = np.array(SP24_PAIRS, np.int64)[which]            # M x C4 x 2
    codes = (pairs[..., 0] | (pairs[..., 1] << 2)).astype(np.uint8)
    E = pack_nibbles(codes) if C4 else np.zeros((M, 0), np.uint8)
    base = (4 * np.arange(C4))[None, :, None]
    pos = (base + pairs).reshape(M, K // 2)
    return store(vals, dtype), E, store(B, dtype), pos

