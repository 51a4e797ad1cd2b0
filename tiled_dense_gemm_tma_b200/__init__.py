"""tiled_dense_gemm_tma_b200 -- tiled dense GEMM for one NVIDIA B200 (sm_100a).

C = epi(A . B) with row-major A (M x K) and B (K x N), epi = identity or
ReLU, in five precisions (fp32 FFMA or TF32, fp16, bf16, the 4-bit-weight
dequantize GEMM, and the FP4-weight (MXFP4) GEMM), plus a 2:4
structured-sparse GEMM on the sparse tensor cores; 16-bit calls also take transposed operands, and
``matmul`` is a differentiable 16-bit product built on them.  All arithmetic runs in hand-written CUDA kernels behind a
C ABI (``include/tg_gemm.h``); this package is a thin ctypes binding that
marshals torch tensors (device memory and streams only) into that ABI.

The binding loads ``libtg_gemm.so`` on first use and raises if it is
missing; there is no CPU or library fallback.
"""
from .binding import (  # noqa: F401
    TgError, gemm_f32, gemm_f16, gemm_bf16, gemm_w4a16, gemm_wfp4, gemm_sp24,
    gemm_bf16_small_m_static,
    matmul, last_device_status,
    lib_path, load_library, EPI_NONE, EPI_RELU, F32_FFMA, F32_TF32,
    tune_set, tune_builtin, tune_query, OPS, PATHS,
)
