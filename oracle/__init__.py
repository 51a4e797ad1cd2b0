"""CPU oracle for the tiled dense GEMM: C = epi(A . B) computed in fp64.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline leg may import this package.  It shares no code
with the CUDA library (``tiled_dense_gemm_tma_b200``) and never imports it.

Each function follows the plain definition of the operation (the scalar
triple loop on the gtnt.cn TileLang tutorial, section 1.1; C = A x B with
row-major A and B on the mhpq.cn TileLang GEMM article, section 2.1; the
ReLU post-processing and the dequantize GEMM on the blog.hotdry.top TileLang
guide; the FP4-weight GEMM named on the krestaai TileLang architecture page,
read as MXFP4 weights with bf16 activations; the 2:4 structured-sparse GEMM
named on the blog.hotdry.top guide, read as the usual compressed values plus
2-bit position codes).  The arithmetic lives in
``oracle.c``; this module only marshals
numpy arrays through ctypes.

Inputs are numpy arrays holding the *stored* values: float32 for fp32,
uint16 bit patterns for fp16 / bf16, uint8 packed bytes for 4-bit weights.
Outputs are float64 arrays (the exact-as-double result), plus rounding
helpers that produce the stored output type with round-to-nearest-even.

Parity of every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, exact rational brute force, an independent numpy
float64 matmul and hand-decoded fixtures in ``tests/golden/``.
"""
import ctypes

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, vp, dp = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p
        for name in ("oracle_gemm_f32", "oracle_gemm_f16", "oracle_gemm_bf16"):
            fn = getattr(lib, name)
            fn.argtypes = [i64, i64, i64, vp, i64, vp, i64, dp, i64, ctypes.c_int]
            fn.restype = None
        lib.oracle_gemm_w4a16.argtypes = [i64, i64, i64, vp, i64, vp, i64, vp, i64,
                                          i64, dp, i64, ctypes.c_int]
        lib.oracle_gemm_w4a16.restype = None
        lib.oracle_dequant_w4.argtypes = [i64, i64, vp, i64, vp, i64, i64, dp, i64]
        lib.oracle_dequant_w4.restype = None
        lib.oracle_gemm_wfp4.argtypes = [i64, i64, i64, vp, i64, vp, i64, vp, i64,
                                         i64, dp, i64, ctypes.c_int]
        lib.oracle_gemm_wfp4.restype = None
        lib.oracle_dequant_fp4.argtypes = [i64, i64, vp, i64, vp, i64, i64, dp, i64]
        lib.oracle_dequant_fp4.restype = None
        lib.oracle_expand_sp24.argtypes = [i64, i64, vp, i64, vp, i64, ctypes.c_int, dp, i64]
        lib.oracle_expand_sp24.restype = None
        lib.oracle_gemm_sp24.argtypes = [i64, i64, i64, vp, i64, vp, i64, vp, i64, ctypes.c_int,
                                         dp, i64, ctypes.c_int]
        lib.oracle_gemm_sp24.restype = None
        lib.oracle_e2m1_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_to_f64.restype = ctypes.c_double
        lib.oracle_e8m0_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e8m0_to_f64.restype = ctypes.c_double
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_round_f16.argtypes = [ctypes.c_double]
        lib.oracle_round_f16.restype = ctypes.c_uint16
        lib.oracle_round_bf16.argtypes = [ctypes.c_double]
        lib.oracle_round_bf16.restype = ctypes.c_uint16
        lib.oracle_round_f32.argtypes = [ctypes.c_double]
        lib.oracle_round_f32.restype = ctypes.c_float
        for name in ("oracle_f16_to_f64_n", "oracle_bf16_to_f64_n",
                     "oracle_round_f16_n", "oracle_round_bf16_n"):
            fn = getattr(lib, name)
            fn.argtypes = [vp, vp, i64]
            fn.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check2d(a, dtype, name):
    if not isinstance(a, np.ndarray) or a.ndim != 2 or a.dtype != dtype:
        raise TypeError(f"{name} must be a 2-D numpy {np.dtype(dtype).name} array")
    if a.strides[1] != a.itemsize or a.strides[0] % a.itemsize:
        raise ValueError(f"{name} must be row-major with unit column stride")
    return a.strides[0] // a.itemsize


def num_threads() -> int:
    """OpenMP threads the oracle uses (set OMP_NUM_THREADS before first load)."""
    return _load().oracle_num_threads()


def _gemm16(fn, A, B, relu):
    lda = _check2d(A, np.uint16, "A")
    ldb = _check2d(B, np.uint16, "B")
    M, K = A.shape
    K2, N = B.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    C = np.empty((M, N), np.float64)
    fn(M, N, K, _ptr(A), lda, _ptr(B), ldb, _ptr(C), N, int(bool(relu)))
    return C


def gemm_f32(A, B, relu=False):
    """fp64 value of epi(A . B) for float32 A (M x K) and B (K x N)."""
    lda = _check2d(A, np.float32, "A")
    ldb = _check2d(B, np.float32, "B")
    M, K = A.shape
    K2, N = B.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    C = np.empty((M, N), np.float64)
    _load().oracle_gemm_f32(M, N, K, _ptr(A), lda, _ptr(B), ldb, _ptr(C), N,
                            int(bool(relu)))
    return C


def gemm_f16(A_bits, B_bits, relu=False):
    """fp64 value of epi(A . B) for fp16 operands given as uint16 bit patterns."""
    return _gemm16(_load().oracle_gemm_f16, A_bits, B_bits, relu)


def gemm_bf16(A_bits, B_bits, relu=False):
    """fp64 value of epi(A . B) for bf16 operands given as uint16 bit patterns."""
    return _gemm16(_load().oracle_gemm_bf16, A_bits, B_bits, relu)


def dequant_w4(Bq, scales, N, group=128):
    """fp64 W (K x N) with W[k, n] = q[k, n] * s[k // group, n]."""
    ldbq = _check2d(Bq, np.uint8, "Bq")
    lds = _check2d(scales, np.uint16, "scales")
    K = Bq.shape[0]
    W = np.empty((K, N), np.float64)
    _load().oracle_dequant_w4(K, N, _ptr(Bq), ldbq, _ptr(scales), lds, group,
                              _ptr(W), N)
    return W


def gemm_w4a16(A_bits, Bq, scales, N, group=128, relu=False):
    """fp64 value of epi(A . W), W the explicitly dequantised 4-bit weight.

    A_bits: M x K fp16 bit patterns.  Bq: K x ceil(N/2) packed bytes (low
    nibble = even column).  scales: (K/group) x N fp16 bit patterns.
    """
    lda = _check2d(A_bits, np.uint16, "A")
    ldbq = _check2d(Bq, np.uint8, "Bq")
    lds = _check2d(scales, np.uint16, "scales")
    M, K = A_bits.shape
    if Bq.shape[0] != K:
        raise ValueError("inner dimensions differ")
    C = np.empty((M, N), np.float64)
    _load().oracle_gemm_w4a16(M, N, K, _ptr(A_bits), lda, _ptr(Bq), ldbq,
                              _ptr(scales), lds, group, _ptr(C), N,
                              int(bool(relu)))
    return C


def e2m1_to_f64(code):
    """Value of one FP4 E2M1 code (0..15)."""
    return _load().oracle_e2m1_to_f64(int(code))


def e8m0_to_f64(e):
    """Value of one E8M0 scale byte: 2^(e - 127), NaN for 255."""
    return _load().oracle_e8m0_to_f64(int(e))


def dequant_fp4(Bq, scales, N, block=32):
    """fp64 W (K x N) with W[k, n] = e2m1(code[k, n]) * e8m0(E[k // block, n])."""
    ldbq = _check2d(Bq, np.uint8, "Bq")
    lds = _check2d(scales, np.uint8, "scales")
    K = Bq.shape[0]
    W = np.empty((K, N), np.float64)
    _load().oracle_dequant_fp4(K, N, _ptr(Bq), ldbq, _ptr(scales), lds, block,
                               _ptr(W), N)
    return W


def gemm_wfp4(A_bits, Bq, scales, N, block=32, relu=False):
    """fp64 value of epi(A . W), W the explicitly dequantised MXFP4 weight.

    A_bits: M x K bf16 bit patterns.  Bq: K x ceil(N/2) bytes of E2M1 codes
    (low nibble = even column).  scales: (K/block) x N E8M0 bytes.
    """
    lda = _check2d(A_bits, np.uint16, "A")
    ldbq = _check2d(Bq, np.uint8, "Bq")
    lds = _check2d(scales, np.uint8, "scales")
    M, K = A_bits.shape
    if Bq.shape[0] != K:
        raise ValueError("inner dimensions differ")
    C = np.empty((M, N), np.float64)
    _load().oracle_gemm_wfp4(M, N, K, _ptr(A_bits), lda, _ptr(Bq), ldbq,
                             _ptr(scales), lds, block, _ptr(C), N, int(bool(relu)))
    return C


def _sp24_args(Ac, E, K, dtype):
    if dtype not in ("f16", "bf16"):
        raise ValueError("dtype must be 'f16' or 'bf16'")
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    ldac = _check2d(Ac, np.uint16, "Ac")
    lde = _check2d(E, np.uint8, "E")
    M = Ac.shape[0]
    if E.shape[0] != M or Ac.shape[1] < K // 2 or E.shape[1] < (K + 7) // 8:
        raise ValueError("Ac must be M x K/2 and E M x ceil(K/8)")
    return M, ldac, lde, int(dtype == "bf16")


def expand_sp24(Ac, E, K, dtype):
    """Dense fp64 A (M x K) of a 2:4 compressed matrix: Ac (M x K/2 16-bit
    bit patterns, the kept values of each chunk of 4 k) and E (M x K/8 bytes,
    a 4-bit code per chunk: bits 0-1 / 2-3 = positions of the first / second
    kept value; even chunk in the low nibble)."""
    M, ldac, lde, bf = _sp24_args(Ac, E, K, dtype)
    A = np.empty((M, K), np.float64)
    _load().oracle_expand_sp24(M, K, _ptr(Ac), ldac, _ptr(E), lde, bf, _ptr(A), K)
    return A


def gemm_sp24(Ac, E, B_bits, dtype, relu=False):
    """fp64 value of epi(A . B) for a 2:4 compressed A (see expand_sp24) and
    a dense B (K x N) of the same 16-bit type, given as bit patterns."""
    K, N = B_bits.shape
    M, ldac, lde, bf = _sp24_args(Ac, E, K, dtype)
    ldb = _check2d(B_bits, np.uint16, "B")
    C = np.empty((M, N), np.float64)
    _load().oracle_gemm_sp24(M, N, K, _ptr(Ac), ldac, _ptr(E), lde, _ptr(B_bits), ldb, bf,
                             _ptr(C), N, int(bool(relu)))
    return C


def _map16(fn_name, bits):
    b = np.ascontiguousarray(bits, np.uint16)
    out = np.empty(b.shape, np.float64)
    getattr(_load(), fn_name)(_ptr(b), _ptr(out), b.size)
    return out


def _round16(fn_name, x):
    a = np.ascontiguousarray(x, np.float64)
    out = np.empty(a.shape, np.uint16)
    getattr(_load(), fn_name)(_ptr(a), _ptr(out), a.size)
    return out


def f16_to_f64(bits):
    """Decode fp16 bit patterns (array) to float64, elementwise."""
    return _map16("oracle_f16_to_f64_n", bits)


def bf16_to_f64(bits):
    """Decode bf16 bit patterns (array) to float64, elementwise."""
    return _map16("oracle_bf16_to_f64_n", bits)


def round_f16(x):
    """Round float64 values to fp16 bit patterns (nearest even)."""
    return _round16("oracle_round_f16_n", x)


def round_bf16(x):
    """Round float64 values to bf16 bit patterns (nearest even)."""
    return _round16("oracle_round_bf16_n", x)


def round_f32(x):
    """Round float64 values to float32 (nearest even)."""
    return np.asarray(x, np.float64).astype(np.float32)
