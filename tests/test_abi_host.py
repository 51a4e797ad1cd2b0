"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/tg_gemm.h declares, and rejects bad arguments before
touching CUDA (nothing is launched, so these run on a machine without GPU)."""
import ctypes
import os
import re

import pytest

from tiled_dense_gemm_tma_b200 import binding, build as tg_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, ALIGN, UNSUP = 0, 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    tg_build.build()
    return binding.load_library()


def test_header_symbols_exported(lib):
    with open(os.path.join(ROOT, "include", "tg_gemm.h")) as f:
        text = f.read()
    declared = set(re.findall(r"\b(tg_\w+)\s*\(", text))
    assert declared == set(binding.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in binding.STATUS.items():
        assert lib.tg_status_string(code).decode() == name
    assert lib.tg_status_string(99).decode() == "TG_ERR_UNKNOWN"


P = 0x10000          # a fake, 16-byte aligned "device" address (never dereferenced)


def _bf16(lib, M, N, K, A=P, lda=None, B=P, ldb=None, C=P, ldc=None, epi=0):
    lda = K if lda is None else lda
    ldb = N if ldb is None else ldb
    ldc = N if ldc is None else ldc
    return lib.tg_gemm_bf16(M, N, K, A, lda, B, ldb, C, ldc, epi, None)


def test_argument_validation_bf16(lib):
    assert _bf16(lib, -1, 8, 8) == INVALID
    assert _bf16(lib, 8, -1, 8) == INVALID
    assert _bf16(lib, 8, 8, -1) == INVALID
    assert _bf16(lib, 8, 8, 8, epi=2) == INVALID
    assert _bf16(lib, 0, 8, 8) == OK               # empty output: nothing to do
    assert _bf16(lib, 8, 0, 8) == OK
    assert _bf16(lib, 8, 8, 8, A=None) == INVALID
    assert _bf16(lib, 8, 8, 8, C=None) == INVALID
    assert _bf16(lib, 8, 8, 8, lda=7) == INVALID
    assert _bf16(lib, 8, 8, 8, ldc=4) == INVALID
    assert _bf16(lib, 8, 8, 8, A=P + 8) == ALIGN
    assert _bf16(lib, 8, 8, 8, C=P + 2) == ALIGN
    assert _bf16(lib, 8, 12, 8, ldb=12, ldc=16) == ALIGN   # 24-byte row pitch
    assert _bf16(lib, 8, 8, 8, lda=12) == ALIGN
    assert _bf16(lib, 1 << 31, 8, 8) == UNSUP


def test_argument_validation_f32_and_f16(lib):
    f = lib.tg_gemm_f32
    assert f(8, 8, 8, P, 8, P, 8, P, 8, 0, 2, None) == INVALID      # bad mode
    assert f(8, 8, 8, P, 6, P, 8, P, 8, 0, 0, None) == INVALID      # lda < K
    assert f(8, 8, 8, P, 10, P, 8, P, 8, 0, 0, None) == ALIGN       # 40-byte pitch
    assert f(8, 0, 8, P, 8, P, 8, P, 8, 0, 1, None) == OK
    g = lib.tg_gemm_f16
    assert g(8, 8, 8, P, 8, P, 8, P + 4, 8, 0, None) == ALIGN
    assert g(8, 8, 8, P, 8, None, 8, P, 8, 0, None) == INVALID


def test_argument_validation_w4a16(lib):
    w = lib.tg_gemm_w4a16
    # M, N, K, A, lda, Bq, ldbq, scales, lds, group, C, ldc, epi, stream
    assert w(4, 32, 256, P, 256, P, 16, P, 32, 64, P, 32, 0, None) == UNSUP     # group 64
    assert w(4, 32, 200, P, 200, P, 16, P, 32, 128, P, 32, 0, None) == UNSUP    # K % 128
    assert w(4, 32, 256, P, 256, P, 8, P, 32, 128, P, 32, 0, None) == INVALID   # ldbq < N/2
    assert w(4, 32, 256, P, 256, P, 24, P, 32, 128, P, 32, 0, None) == ALIGN    # ldbq % 16
    assert w(4, 32, 256, P, 256, P, 16, P + 2, 32, 128, P, 32, 0, None) == ALIGN
    assert w(4, 32, 256, P, 256, P, 16, None, 32, 128, P, 32, 0, None) == INVALID
    assert w(0, 32, 256, P, 256, P, 16, P, 32, 128, P, 32, 0, None) == OK
    assert w(4, 32, 256, P, 256, P, 16, P, 32, 128, P, 32, 3, None) == INVALID


def test_argument_validation_wfp4(lib):
    w = lib.tg_gemm_wfp4
    # M, N, K, A, lda, Bq, ldbq, scales, lds (bytes), block, C, ldc, epi, stream
    assert w(4, 32, 256, P, 256, P, 16, P, 32, 16, P, 32, 0, None) == UNSUP     # block 16
    assert w(4, 32, 256, P, 256, P, 8, P, 32, 32, P, 32, 0, None) == INVALID    # ldbq < N/2
    assert w(4, 32, 256, P, 256, P, 16, P, 16, 32, P, 32, 0, None) == INVALID   # lds < N bytes
    assert w(4, 32, 256, P, 256, P, 24, P, 32, 32, P, 32, 0, None) == ALIGN     # ldbq % 16
    assert w(4, 40, 256, P, 256, P, 32, P, 40, 32, P, 40, 0, None) == ALIGN     # lds % 16
    assert w(4, 32, 256, P, 256, P, 16, P + 8, 32, 32, P, 32, 0, None) == ALIGN
    assert w(4, 32, 256, P, 256, P, 16, None, 32, 32, P, 32, 0, None) == INVALID
    assert w(0, 32, 256, P, 256, P, 16, P, 32, 32, P, 32, 0, None) == OK
    assert w(4, 32, 256, P, 256, P, 16, P, 32, 32, P, 32, 2, None) == INVALID
    huge = (1 << 62) + 8
    assert w(4, 32, 256, P, 256, P, 16, P, huge, 32, P, 32, 0, None) == UNSUP   # lds
    assert w(4, 32, 256, P, 256, P, 1 << 40, P, 32, 32, P, 32, 0, None) == UNSUP


def test_argument_validation_sp24(lib):
    for f in (lib.tg_gemm_sp24_f16, lib.tg_gemm_sp24_bf16):
        # M, N, K, Ac, ldac, E, lde (bytes), B, ldb, C, ldc, epi, stream
        assert f(8, 8, 30, P, 16, P, 16, P, 8, P, 8, 0, None) == UNSUP        # K % 4
        assert f(8, 8, 64, P, 24, P, 16, P, 8, P, 8, 0, None) == INVALID      # ldac < K/2
        assert f(8, 8, 256, P, 128, P, 16, P, 8, P, 8, 0, None) == INVALID    # lde < K/8
        assert f(8, 8, 64, P, 36, P, 16, P, 8, P, 8, 0, None) == ALIGN        # 72-byte pitch
        assert f(8, 8, 64, P, 32, P, 24, P, 8, P, 8, 0, None) == ALIGN        # lde % 16
        assert f(8, 8, 64, P, 32, None, 16, P, 8, P, 8, 0, None) == INVALID
        assert f(8, 8, 64, P, 32, P + 4, 16, P, 8, P, 8, 0, None) == ALIGN
        assert f(0, 8, 64, P, 32, P, 16, P, 8, P, 8, 0, None) == OK
        assert f(8, 8, 64, P, 32, P, 16, P, 8, P, 8, 3, None) == INVALID
        assert f(8, 8, 64, P, 32, P, (1 << 62) + 16, P, 8, P, 8, 0, None) == UNSUP


def test_row_pitch_limits(lib):
    """Row pitches of 2^40 bytes or more are refused before any product
    ld * sizeof(element) is formed, so even pitches near 2^63 are reported
    as TG_ERR_UNSUPPORTED rather than wrapping into a small value."""
    huge = (1 << 62) + 8                       # * 2 or * 4 would overflow int64
    at_limit = (1 << 39)                       # 2^40 bytes of bf16
    assert _bf16(lib, 8, 8, 8, ldc=at_limit) == UNSUP
    assert _bf16(lib, 8, 8, 8, lda=huge) == UNSUP
    assert _bf16(lib, 8, 8, 8, ldb=huge) == UNSUP
    assert _bf16(lib, 8, 8, 8, ldc=huge) == UNSUP
    f = lib.tg_gemm_f32
    assert f(8, 8, 8, P, 1 << 38, P, 8, P, 8, 0, 0, None) == UNSUP   # 2^40 bytes of fp32
    w = lib.tg_gemm_w4a16
    assert w(4, 32, 256, P, 256, P, 1 << 40, P, 32, 128, P, 32, 0, None) == UNSUP   # ldbq
    assert w(4, 32, 256, P, 256, P, 16, P, huge, 128, P, 32, 0, None) == UNSUP      # lds
    assert w(4, 32, 256, P, huge, P, 16, P, 32, 128, P, 32, 0, None) == UNSUP       # lda
    assert w(4, 32, 256, P, 256, P, 16, P, 32, 128, P, huge, 0, None) == UNSUP      # ldc
    s = lib.tg_gemm_bf16_small_m_static
    for big in (1 << 40, huge):
        assert s(16, 8, 8, P, big, P, 8, P, 8, 0, None) == UNSUP                    # lda
        assert s(16, 8, 8, P, 8, P, big, P, 8, 0, None) == UNSUP                    # ldb
        assert s(16, 8, 8, P, 8, P, 8, P, big, 0, None) == UNSUP                    # ldc


def test_argument_validation_small_m_static(lib):
    """The entry point that never allocates runs the same checks as
    tg_gemm_bf16 before any CUDA call, plus its own M <= 128 limit."""
    s = lib.tg_gemm_bf16_small_m_static
    assert s(-1, 8, 8, P, 8, P, 8, P, 8, 0, None) == INVALID
    assert s(16, 8, 8, P, 8, P, 8, P, 8, 2, None) == INVALID            # bad epilogue
    assert s(16, 8, 8, None, 8, P, 8, P, 8, 0, None) == INVALID
    assert s(16, 8, 8, P, 7, P, 8, P, 8, 0, None) == INVALID            # lda < K
    assert s(16, 8, 8, P + 8, 8, P, 8, P, 8, 0, None) == ALIGN
    assert s(16, 8, 8, P, 12, P, 8, P, 8, 0, None) == ALIGN             # 24-byte pitch
    assert s(0, 8, 8, P, 8, P, 8, P, 8, 0, None) == OK
    assert s(129, 8, 8, P, 8, P, 8, P, 8, 0, None) == UNSUP             # M above 128
    assert s(16, 1 << 31, 8, P, 8, P, 1 << 31, P, 1 << 31, 0, None) == UNSUP


def test_ffma_size_limits_refused_before_any_cuda_call(lib):
    """The fp32 FFMA kernel's own limits (a 32-bit output pitch, at most
    65535 rows of 128-row tiles) are refused before the library touches
    CUDA, so they read TG_ERR_UNSUPPORTED even without a device."""
    f = lib.tg_gemm_f32
    assert f(8, 8, 8, P, 8, P, 8, P, 1 << 31, 0, 0, None) == UNSUP
    M = 65535 * 128 + 1
    assert f(M, 8, 8, P, 8, P, 8, P, 8, 0, 0, None) == UNSUP


def test_valid_calls_without_a_device_report_no_device(lib):
    """On a machine with no GPU a well-formed call gets past validation and
    must report TG_ERR_NO_DEVICE (no CPU fallback, no crash).  The fake
    pointers must never reach a kernel, so this runs only where the library
    itself sees no device."""
    if lib.tg_num_sms() >= 0:
        pytest.skip("a CUDA device is present")
    NODEV = 6
    assert _bf16(lib, 64, 64, 64) == NODEV
    assert lib.tg_gemm_f16(64, 64, 64, P, 64, P, 64, P, 64, 0, None) == NODEV
    for mode in (0, 1):
        assert lib.tg_gemm_f32(64, 64, 64, P, 64, P, 64, P, 64, 0, mode, None) == NODEV
    assert lib.tg_gemm_w4a16(4, 32, 256, P, 256, P, 16, P, 32, 128, P, 32, 0, None) == NODEV
    assert lib.tg_gemm_wfp4(4, 32, 200, P, 200, P, 16, P, 32, 32, P, 32, 0, None) == NODEV
    assert lib.tg_gemm_sp24_bf16(8, 8, 64, P, 32, P, 16, P, 8, P, 8, 0, None) == NODEV
    assert lib.tg_gemm_bf16_ex(64, 64, 64, P, 64, 1, P, 64, 1, P, 64, 0, None) == NODEV
    assert lib.tg_gemm_f16_ex(64, 64, 64, P, 64, 0, P, 64, 1, P, 64, 0, None) == NODEV
    assert lib.tg_gemm_bf16_small_m_static(16, 64, 64, P, 64, P, 64, P, 64, 0, None) == NODEV
    # K == 0 writes C = 0 with a device memset: also no device here
    assert _bf16(lib, 8, 8, 0) == NODEV


C_PROGRAM = r"""
#include <stdio.h>
#include "tg_gemm.h"
/* Every entry point, called from plain C with arguments that fail
   validation: prints each status so the test can check them. */
int main(void) {
    printf("%d\n", tg_gemm_f32(-1, 8, 8, 0, 8, 0, 8, 0, 8, TG_EPI_NONE, TG_F32_FFMA, 0));
    printf("%d\n", tg_gemm_f16(8, 8, 8, 0, 8, 0, 8, 0, 8, TG_EPI_NONE, 0));
    printf("%d\n", tg_gemm_bf16(8, 8, 8, 0, 8, 0, 8, 0, 8, 7, 0));
    printf("%d\n", tg_gemm_f16_ex(8, 8, 8, 0, 8, 2, 0, 8, 0, 0, 8, TG_EPI_NONE, 0));
    printf("%d\n", tg_gemm_bf16_ex(8, 8, 8, 0, 8, 0, 0, 8, 3, 0, 8, TG_EPI_NONE, 0));
    printf("%d\n", tg_gemm_w4a16(4, 32, 256, 0, 256, 0, 16, 0, 32, 64, 0, 32, TG_EPI_NONE, 0));
    printf("%d\n", tg_gemm_bf16_small_m_static(0, 8, 8, 0, 8, 0, 8, 0, 8, TG_EPI_NONE, 0));
    printf("%d\n", tg_gemm_wfp4(4, 32, 256, 0, 256, 0, 16, 0, 32, 16, 0, 32, TG_EPI_NONE, 0));
    printf("%s\n", tg_status_string(TG_ERR_ALIGNMENT));
    return 0;
}
"""


def test_header_is_plain_c_and_links(tmp_path):
    """include/tg_gemm.h compiles as strict C99 and a C program links
    libtg_gemm.so and gets the documented status codes back."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "abi_check.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi_check"
    libdir = os.path.dirname(binding.lib_path())
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-L", libdir, "-ltg_gemm",
                    "-Wl,-rpath," + libdir, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    # negative M; null pointers; bad epilogue; bad trans flags (x2); group 64; M == 0;
    # FP4 block 16
    assert out[:8] == [str(c) for c in (INVALID, INVALID, INVALID, INVALID, INVALID, UNSUP, OK,
                                        UNSUP)]
    assert out[8] == "TG_ERR_ALIGNMENT"


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_HERE", str(tmp_path))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(ImportError):
        binding.load_library()


def _bf16_ex(lib, M, N, K, ta, tb, lda, ldb, ldc=None, A=P, B=P, C=P):
    ldc = N if ldc is None else ldc
    return lib.tg_gemm_bf16_ex(M, N, K, A, lda, ta, B, ldb, tb, C, ldc, 0, None)


def test_argument_validation_transposed(lib):
    # stored A is K x M when transposed: its pitch must cover M, not K
    assert _bf16_ex(lib, 64, 32, 16, 1, 0, lda=56, ldb=32) == INVALID    # lda < M
    assert _bf16_ex(lib, 64, 32, 16, 0, 1, lda=16, ldb=8) == INVALID     # ldb < K
    assert _bf16_ex(lib, 64, 32, 16, 2, 0, lda=64, ldb=32) == INVALID    # flag not 0 / 1
    assert _bf16_ex(lib, 64, 32, 16, 0, -1, lda=16, ldb=16) == INVALID
    assert _bf16_ex(lib, 64, 32, 16, 1, 1, lda=64, ldb=20) == ALIGN      # 40-byte B pitch
    assert _bf16_ex(lib, 0, 32, 16, 1, 1, lda=64, ldb=16) == OK          # empty output
    assert lib.tg_gemm_f16_ex(64, 32, 16, P, 60, 1, P, 32, 0, P, 32, 0, None) == INVALID


def test_tuning_table_rules(lib):
    """tg_tune_set validates every rule before installing any, run-time rules
    are consulted before the built-in ones in the order given, and a call
    shape no rule covers gets the all-default rule (no CUDA call needed)."""
    from tiled_dense_gemm_tma_b200 import binding as b
    b.tune_set([])
    try:
        builtin = b.tune_builtin()
        for r in builtin:
            assert b.tune_query(r["op"], r["m_lo"], r["n_lo"]) == r
        rules = [{"op": "bf16", "path": "small_m", "m_lo": 5, "m_hi": 64, "ctas": 100},
                 {"op": "bf16", "path": "cta_pair", "m_lo": 1, "m_hi": 1 << 40, "stages": 4,
                  "group_m": 4},
                 {"op": "f32_ffma", "splits": 3},
                 {"op": "f32_tf32", "path": "one_cta", "m_lo": 129, "m_hi": 4096},
                 {"op": "f32_tf32", "path": "cta_pair", "m_lo": 1, "m_hi": 128}]
        b.tune_set(rules)
        q = b.tune_query("bf16", 16, 8192)
        assert (q["path"], q["ctas"]) == (b.PATHS["small_m"], 100)        # first match wins
        q = b.tune_query("bf16", 65, 8192)
        assert (q["path"], q["stages"], q["group_m"]) == (b.PATHS["cta_pair"], 4, 4)
        assert b.tune_query("f32_ffma", 1024, 1024)["splits"] == 3
        # TF32 runs on either tensor-core kernel, by rule
        assert b.tune_query("f32_tf32", 4096, 4096)["path"] == b.PATHS["one_cta"]
        assert b.tune_query("f32_tf32", 100, 4096)["path"] == b.PATHS["cta_pair"]
        # malformed rules: nothing changes
        bad = [{"op": "bf16", "path": "cuda_core", "m_hi": 5},       # CUDA-core kernel: M <= 4
               {"op": "wfp4", "path": "cuda_core", "m_hi": 5},        # CUDA-core FP4 kernel: M <= 4
               {"op": "bf16", "path": "small_m", "m_hi": 129},        # small-M kernel: M <= 128
               {"op": "f32_ffma", "path": "one_cta"},                 # fp32 FFMA has one kernel
               {"op": "f32_ffma", "path": "cta_pair"},
               {"op": "f32_tf32", "path": "small_m", "m_hi": 128},    # no fp32 small-M kernel
               {"op": "f32_tf32", "path": "cuda_core", "m_hi": 4},
               {"op": "bf16", "splits": 2},                           # split count: FFMA only
               {"op": "w4a16", "stages": 4},                          # ring depth: 16-bit pair only
               {"op": "bf16", "stages": 5},
               {"op": "bf16", "m_lo": 10, "m_hi": 9},
               {"op": 9}, {"op": "bf16", "path": 7}, {"op": "bf16", "ctas": -1}]
        for r in bad:
            with pytest.raises(b.TgError):
                b.tune_set([rules[0], r])
            assert b.tune_query("bf16", 16, 8192)["ctas"] == 100
        assert lib.tg_tune_set(None, 1) == INVALID
        assert lib.tg_tune_set(None, 0) == OK
        q = b.tune_query("bf16", 16, 8192)
        assert q["ctas"] == 0 or q in builtin
    finally:
        b.tune_set([])
