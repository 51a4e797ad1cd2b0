"""ctypes binding of the C ABI declared in include/tg_gemm.h.

Argument marshalling only: every step of the GEMM runs in the CUDA kernels
of ``libtg_gemm.so``.  Torch is used for device memory and streams.  If the
library is missing, the first call raises; there is no fallback.
"""
import contextlib
import ctypes
import os
import threading

LIB_NAME = "libtg_gemm.so"
_HERE = os.path.dirname(os.path.abspath(__file__))

EPI_NONE, EPI_RELU = 0, 1
F32_FFMA, F32_TF32 = 0, 1

STATUS = {0: "TG_OK", 1: "TG_ERR_INVALID_ARG", 2: "TG_ERR_ALIGNMENT",
          3: "TG_ERR_UNSUPPORTED", 4: "TG_ERR_CUDA", 5: "TG_ERR_TIMEOUT",
          6: "TG_ERR_NO_DEVICE"}

# Every symbol include/tg_gemm.h declares.
EXPORTS = ("tg_gemm_f32", "tg_gemm_f16", "tg_gemm_bf16", "tg_gemm_w4a16", "tg_gemm_wfp4",
           "tg_gemm_f16_ex", "tg_gemm_bf16_ex", "tg_gemm_bf16_small_m_static",
           "tg_gemm_sp24_f16", "tg_gemm_sp24_bf16",
           "tg_tune_set", "tg_tune_builtin", "tg_tune_query",
           "tg_status_string", "tg_last_device_status", "tg_num_sms")

# Tuning table (include/tg_gemm.h: tg_tune_rule): operations and kernel paths.
OPS = {"bf16": 0, "f16": 1, "w4a16": 2, "wfp4": 3, "f32_ffma": 4, "f32_tf32": 5}
PATHS = {"auto": 0, "cuda_core": 1, "small_m": 2, "cta_pair": 3, "one_cta": 4}


class TuneRule(ctypes.Structure):
    """tg_tune_rule: which kernel family and launch shape a call uses."""
    _fields_ = [("op", ctypes.c_int32), ("path", ctypes.c_int32),
                ("m_lo", ctypes.c_int64), ("m_hi", ctypes.c_int64),
                ("n_lo", ctypes.c_int64), ("n_hi", ctypes.c_int64),
                ("ctas", ctypes.c_int32), ("group_m", ctypes.c_int32),
                ("splits", ctypes.c_int32), ("stages", ctypes.c_int32)]

_lib = None
_lock = threading.Lock()


class TgError(RuntimeError):
    """A non-OK tg_status returned by the library."""

    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)}")


def lib_path():
    return os.path.join(_HERE, LIB_NAME)


def load_library():
    """Load libtg_gemm.so (built in-tree) and declare its signatures."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = lib_path()
        if not os.path.exists(path):
            raise ImportError(f"{LIB_NAME} is not built (expected at {path}); "
                              "run tiled_dense_gemm_tma_b200/build.py")
        lib = ctypes.CDLL(path)
        i64, vp, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        lib.tg_gemm_f32.argtypes = [i64, i64, i64, vp, i64, vp, i64, vp, i64, ci, ci, vp]
        for name in ("tg_gemm_f16", "tg_gemm_bf16", "tg_gemm_bf16_small_m_static"):
            getattr(lib, name).argtypes = [i64, i64, i64, vp, i64, vp, i64, vp, i64, ci, vp]
        for name in ("tg_gemm_w4a16", "tg_gemm_wfp4"):
            getattr(lib, name).argtypes = [i64, i64, i64, vp, i64, vp, i64, vp, i64, ci,
                                           vp, i64, ci, vp]
        for name in ("tg_gemm_sp24_f16", "tg_gemm_sp24_bf16"):
            getattr(lib, name).argtypes = [i64, i64, i64, vp, i64, vp, i64, vp, i64, vp, i64, ci, vp]
            getattr(lib, name).restype = ci
        for name in ("tg_gemm_f16_ex", "tg_gemm_bf16_ex"):
            getattr(lib, name).argtypes = [i64, i64, i64, vp, i64, ci, vp, i64, ci, vp, i64, ci, vp]
        for name in ("tg_gemm_f32", "tg_gemm_f16", "tg_gemm_bf16", "tg_gemm_w4a16",
                     "tg_gemm_wfp4", "tg_gemm_f16_ex", "tg_gemm_bf16_ex",
                     "tg_gemm_bf16_small_m_static", "tg_last_device_status"):
            getattr(lib, name).restype = ci
        lib.tg_status_string.argtypes = [ci]
        lib.tg_status_string.restype = ctypes.c_char_p
        lib.tg_last_device_status.argtypes = [vp]
        lib.tg_num_sms.argtypes = []
        lib.tg_num_sms.restype = ci
        lib.tg_tune_set.argtypes = [ctypes.POINTER(TuneRule), ci]
        lib.tg_tune_set.restype = ci
        lib.tg_tune_builtin.argtypes = [ctypes.POINTER(TuneRule), ci]
        lib.tg_tune_builtin.restype = ci
        lib.tg_tune_query.argtypes = [ci, i64, i64, ctypes.POINTER(TuneRule)]
        lib.tg_tune_query.restype = ci
        _lib = lib
        return lib


def _stream_handle(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _require_cuda(device, *named):
    """Every tensor on `device`, a CUDA device: the kernels run on the device
    that holds the operands and take raw device pointers."""
    for t, n in named:
        if not t.is_cuda:
            raise ValueError(f"{n} must be a CUDA tensor")
        if t.device != device:
            raise ValueError(f"{n} is on {t.device}, the operands on {device}")


def _device_ctx(t):
    """Make t's device current for the call (the library launches on the
    current device; the default stream is that device's current stream)."""
    if not t.is_cuda:
        return contextlib.nullcontext()
    import torch
    return torch.cuda.device(t.device)


def _ld(t, name):
    """Row pitch (elements) of a row-major 2-D tensor view."""
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D")
    if t.stride(1) != 1 and t.shape[1] > 1:
        raise ValueError(f"{name} must be row-major (unit column stride)")
    return t.stride(0)


def _check(code, what):
    if code != 0:
        raise TgError(code, what)


def empty_out(M, N, dtype, device):
    """An M x N output view whose row pitch is a multiple of 16 bytes."""
    import torch
    per = 16 // torch.tensor([], dtype=dtype).element_size()
    ld = max(per, -(-N // per) * per)
    return torch.empty((M, ld), dtype=dtype, device=device)[:, :N]


def _mk(A, B, C, dtype, out_dtype, trans_a=False, trans_b=False):
    if A.dim() != 2 or B.dim() != 2:
        raise ValueError("A and B must be 2-D")
    M, K = A.shape[::-1] if trans_a else A.shape
    K2, N = B.shape[::-1] if trans_b else B.shape
    if K != K2:
        raise ValueError(f"inner dimensions differ: {K} vs {K2}")
    for t, n in ((A, "A"), (B, "B")):
        if t.dtype != dtype:
            raise TypeError(f"{n} must be {dtype}")
    _require_cuda(A.device, (A, "A"), (B, "B"))
    if C is None:
        C = empty_out(M, N, out_dtype, A.device)
    elif C.shape != (M, N) or C.dtype != out_dtype:
        raise ValueError("C has the wrong shape or dtype")
    _require_cuda(A.device, (C, "C"))
    return M, N, K, C


def gemm_f32(A, B, C=None, relu=False, mode=F32_FFMA, stream=None):
    """C = epi(A @ B) for float32 CUDA tensors; mode F32_FFMA or F32_TF32."""
    import torch
    lib = load_library()
    M, N, K, C = _mk(A, B, C, torch.float32, torch.float32)
    with _device_ctx(A):
        code = lib.tg_gemm_f32(M, N, K, A.data_ptr(), _ld(A, "A"), B.data_ptr(), _ld(B, "B"),
                               C.data_ptr(), _ld(C, "C"), EPI_RELU if relu else EPI_NONE,
                               mode, _stream_handle(stream))
    _check(code, "tg_gemm_f32")
    return C


def _gemm16(name, dtype, A, B, C, relu, stream, trans_a, trans_b):
    lib = load_library()
    M, N, K, C = _mk(A, B, C, dtype, dtype, trans_a, trans_b)
    epi = EPI_RELU if relu else EPI_NONE
    with _device_ctx(A):
        if trans_a or trans_b:
            name += "_ex"
            code = getattr(lib, name)(M, N, K, A.data_ptr(), _ld(A, "A"), int(trans_a),
                                      B.data_ptr(), _ld(B, "B"), int(trans_b),
                                      C.data_ptr(), _ld(C, "C"), epi, _stream_handle(stream))
        else:
            code = getattr(lib, name)(M, N, K, A.data_ptr(), _ld(A, "A"), B.data_ptr(),
                                      _ld(B, "B"), C.data_ptr(), _ld(C, "C"), epi,
                                      _stream_handle(stream))
    _check(code, name)
    return C


def gemm_f16(A, B, C=None, relu=False, stream=None, trans_a=False, trans_b=False):
    """C = epi(op(A) @ op(B)) for float16 CUDA tensors, fp32 accumulation.

    op(A) = A, or A.T when trans_a (A then holds the K x M matrix); op(B) =
    B, or B.T when trans_b (B then holds N x K)."""
    import torch
    return _gemm16("tg_gemm_f16", torch.float16, A, B, C, relu, stream, trans_a, trans_b)


def gemm_bf16(A, B, C=None, relu=False, stream=None, trans_a=False, trans_b=False):
    """C = epi(op(A) @ op(B)) for bfloat16 CUDA tensors, fp32 accumulation
    (op as in gemm_f16)."""
    import torch
    return _gemm16("tg_gemm_bf16", torch.bfloat16, A, B, C, relu, stream, trans_a, trans_b)


def _row_major(t):
    return t.stride(1) == 1 or t.shape[1] <= 1


def _stored(u):
    """How the logical 2-D matrix u reaches the kernels: (storage, transposed)
    with u == storage or u == storage.T and the storage row-major.  A
    transposed view (e.g. W.T of a row-major W) needs no copy.  Where both
    readings hold, the one with a 16-byte row pitch wins, the plain one
    first; a view that is neither is copied to a contiguous tensor."""
    cands = []
    if _row_major(u) and u.stride(0) >= u.shape[1]:
        cands.append((u, False))
    v = u.t()
    if _row_major(v) and v.stride(0) >= v.shape[1]:
        cands.append((v, True))
    for st, tr in cands:
        if (st.stride(0) * st.element_size()) % 16 == 0:
            return st, tr
    if cands:
        return cands[0]
    return u.contiguous(), False


def _autograd_matmul():
    import torch

    class _Matmul(torch.autograd.Function):
        """C = A @ B on this library's 16-bit kernels, with the backward
        products dA = dC @ B^T and dB = A^T @ dC.  Every operand, the
        gradient included, is passed as it is stored: a transposed view
        becomes a transposed-operand call, not a copy."""

        @staticmethod
        def forward(ctx, A, B):
            ctx.save_for_backward(A, B)
            fn = gemm_bf16 if A.dtype == torch.bfloat16 else gemm_f16
            a, ta = _stored(A)
            b, tb = _stored(B)
            return fn(a, b, trans_a=ta, trans_b=tb)

        @staticmethod
        def backward(ctx, dC):
            A, B = ctx.saved_tensors
            fn = gemm_bf16 if A.dtype == torch.bfloat16 else gemm_f16
            g, tg = _stored(dC)
            dA = dB = None
            if ctx.needs_input_grad[0]:
                x, tx = _stored(B.t())
                dA = fn(g, x, trans_a=tg, trans_b=tx)
            if ctx.needs_input_grad[1]:
                y, ty = _stored(A.t())
                dB = fn(y, g, trans_a=ty, trans_b=tg)
            return dA, dB

    return _Matmul


_MATMUL = None


def matmul(A, B):
    """Differentiable C = A @ B for 2-D float16 / bfloat16 CUDA tensors.

    A and B may be row-major or transposed views of row-major storage (such
    as W.T for a linear layer's out x in weight W); both reach the kernels
    without a copy."""
    global _MATMUL
    if _MATMUL is None:
        _MATMUL = _autograd_matmul()
    return _MATMUL.apply(A, B)


def gemm_w4a16(A, Bq, scales, N, C=None, group_size=128, relu=False, stream=None):
    """C = epi(A @ W), W[k, n] = q[k, n] * scales[k // group_size, n].

    A: M x K float16; Bq: K x ldbq uint8 (packed, low nibble = even column);
    scales: (K // group_size) x N float16; N: number of output columns.
    """
    import torch
    lib = load_library()
    if A.dtype != torch.float16 or scales.dtype != torch.float16 or Bq.dtype != torch.uint8:
        raise TypeError("A and scales must be float16, Bq uint8")
    if A.dim() != 2 or Bq.dim() != 2 or scales.dim() != 2:
        raise ValueError("A, Bq and scales must be 2-D")
    M, K = A.shape
    if Bq.shape[0] != K:
        raise ValueError("Bq must have K rows")
    _require_cuda(A.device, (A, "A"), (Bq, "Bq"), (scales, "scales"))
    if C is None:
        C = empty_out(M, N, torch.float16, A.device)
    elif C.shape != (M, N) or C.dtype != torch.float16:
        raise ValueError("C has the wrong shape or dtype")
    _require_cuda(A.device, (C, "C"))
    with _device_ctx(A):
        code = lib.tg_gemm_w4a16(M, N, K, A.data_ptr(), _ld(A, "A"), Bq.data_ptr(),
                                 _ld(Bq, "Bq"), scales.data_ptr(), _ld(scales, "scales"),
                                 group_size, C.data_ptr(), _ld(C, "C"),
                                 EPI_RELU if relu else EPI_NONE, _stream_handle(stream))
    _check(code, "tg_gemm_w4a16")
    return C


def gemm_wfp4(A, Bq, scales, N, C=None, block_size=32, relu=False, stream=None):
    """C = epi(A @ W), W[k, n] = e2m1(code[k, n]) * 2^(scales[k // 32, n] - 127).

    A: M x K bfloat16; Bq: K x ldbq uint8 (E2M1 codes, low nibble = even
    column); scales: ceil(K / 32) x N uint8 E8M0 exponents; N: number of
    output columns.  C is M x N bfloat16.
    """
    import torch
    lib = load_library()
    if A.dtype != torch.bfloat16 or Bq.dtype != torch.uint8 or scales.dtype != torch.uint8:
        raise TypeError("A must be bfloat16, Bq and scales uint8")
    if A.dim() != 2 or Bq.dim() != 2 or scales.dim() != 2:
        raise ValueError("A, Bq and scales must be 2-D")
    M, K = A.shape
    if Bq.shape[0] != K:
        raise ValueError("Bq must have K rows")
    _require_cuda(A.device, (A, "A"), (Bq, "Bq"), (scales, "scales"))
    if C is None:
        C = empty_out(M, N, torch.bfloat16, A.device)
    elif C.shape != (M, N) or C.dtype != torch.bfloat16:
        raise ValueError("C has the wrong shape or dtype")
    _require_cuda(A.device, (C, "C"))
    with _device_ctx(A):
        code = lib.tg_gemm_wfp4(M, N, K, A.data_ptr(), _ld(A, "A"), Bq.data_ptr(), _ld(Bq, "Bq"),
                                scales.data_ptr(), _ld(scales, "scales"), block_size,
                                C.data_ptr(), _ld(C, "C"), EPI_RELU if relu else EPI_NONE,
                                _stream_handle(stream))
    _check(code, "tg_gemm_wfp4")
    return C


def gemm_sp24(Ac, E, B, C=None, relu=False, stream=None):
    """C = epi(A @ B) for a 2:4 structured-sparse A given compressed.

    Ac: M x K/2 float16 or bfloat16 (the two kept values of every chunk of 4
    consecutive k, in increasing k); E: M x ceil(K/8) uint8 position codes
    (per chunk 4 bits, bits 0-1 / 2-3 = positions of the first / second kept
    value, even chunk in the low nibble); B: K x N of Ac's dtype.  K is taken
    from B and must be a multiple of 4.
    """
    import torch
    lib = load_library()
    if Ac.dtype not in (torch.float16, torch.bfloat16) or B.dtype != Ac.dtype:
        raise TypeError("Ac and B must be float16 or bfloat16, the same")
    if E.dtype != torch.uint8:
        raise TypeError("E must be uint8")
    if Ac.dim() != 2 or E.dim() != 2 or B.dim() != 2:
        raise ValueError("Ac, E and B must be 2-D")
    K, N = B.shape
    M = Ac.shape[0]
    if Ac.shape[1] != K // 2 or E.shape[0] != M or E.shape[1] < (K + 7) // 8:
        raise ValueError("Ac must be M x K/2 and E M x ceil(K/8)")
    _require_cuda(Ac.device, (Ac, "Ac"), (E, "E"), (B, "B"))
    if C is None:
        C = empty_out(M, N, Ac.dtype, Ac.device)
    elif C.shape != (M, N) or C.dtype != Ac.dtype:
        raise ValueError("C has the wrong shape or dtype")
    _require_cuda(Ac.device, (C, "C"))
    name = "tg_gemm_sp24_bf16" if Ac.dtype == torch.bfloat16 else "tg_gemm_sp24_f16"
    with _device_ctx(Ac):
        code = getattr(lib, name)(M, N, K, Ac.data_ptr(), _ld(Ac, "Ac"), E.data_ptr(), _ld(E, "E"),
                                  B.data_ptr(), _ld(B, "B"), C.data_ptr(), _ld(C, "C"),
                                  EPI_RELU if relu else EPI_NONE, _stream_handle(stream))
    _check(code, name)
    return C


def gemm_bf16_small_m_static(A, B, C=None, relu=False, stream=None):
    """bf16 GEMM for M <= 128 whose scratch is a fixed device array of the
    library: the call never allocates device memory (C must then be given
    by a caller that cannot allocate)."""
    import torch
    lib = load_library()
    M, N, K, C = _mk(A, B, C, torch.bfloat16, torch.bfloat16)
    with _device_ctx(A):
        code = lib.tg_gemm_bf16_small_m_static(M, N, K, A.data_ptr(), _ld(A, "A"), B.data_ptr(),
                                               _ld(B, "B"), C.data_ptr(), _ld(C, "C"),
                                               EPI_RELU if relu else EPI_NONE,
                                               _stream_handle(stream))
    _check(code, "tg_gemm_bf16_small_m_static")
    return C


def last_device_status(stream=None):
    """Synchronise the stream and return (and clear) the device status word."""
    return load_library().tg_last_device_status(_stream_handle(stream))


_MAX_I64 = (1 << 63) - 1


def _rule_of(d):
    """A TuneRule from a dict: op and path by name or number, ranges default
    to everything, knobs to 0 (the library's default)."""
    op = OPS.get(d["op"], d["op"])
    path = PATHS.get(d.get("path", 0), d.get("path", 0))
    return TuneRule(op, path, d.get("m_lo", 1), d.get("m_hi", _MAX_I64), d.get("n_lo", 1),
                    d.get("n_hi", _MAX_I64), d.get("ctas", 0), d.get("group_m", 0),
                    d.get("splits", 0), d.get("stages", 0))


def _dict_of(r):
    return {f: getattr(r, f) for f, _ in TuneRule._fields_}


def tune_set(rules):
    """Install run-time tuning rules (list of dicts, see _rule_of), consulted
    before the built-in ones; an empty list clears them."""
    lib = load_library()
    arr = (TuneRule * max(1, len(rules)))(*[_rule_of(d) for d in rules])
    _check(lib.tg_tune_set(arr, len(rules)), "tg_tune_set")


def tune_builtin():
    """The built-in tuning rules, as dicts."""
    lib = load_library()
    n = lib.tg_tune_builtin(None, 0)
    arr = (TuneRule * max(1, n))()
    lib.tg_tune_builtin(arr, n)
    return [_dict_of(arr[i]) for i in range(n)]


def tune_query(op, M, N):
    """The rule a call of `op` (name or number) with these M and N uses."""
    lib = load_library()
    r = TuneRule()
    _check(lib.tg_tune_query(OPS.get(op, op), M, N, ctypes.byref(r)), "tg_tune_query")
    return _dict_of(r)
