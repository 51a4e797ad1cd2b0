"""GPU parity of calls whose kernel family and launch shape come from the
tuning table (tg_tune_set): every path a rule can force, CTA counts below
the SM count (fewer stream-K ranges, fewer persistent CTAs), other raster
band heights, the shallower CTA-pair ring and forced fp32 split counts must
still match the fp64 oracle at the tolerances of the plain calls; a rule
that only reorders tiles (band height, ring depth, CTA count of a tiled
kernel) must give bit-identical results.
"""
import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth
from gpu_util import to_dev, from_dev, decode16, guarded_out, check_guard, assert_close, rel_frob

pytestmark = pytest.mark.gpu


@pytest.fixture
def tg():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_dense_gemm_tma_b200 as tg
    tg.load_library()
    tg.tune_set([])
    yield tg
    tg.tune_set([])


def _bf16(tg, A, B):
    import torch
    M, N = A.shape[0], B.shape[1]
    big, C, pad = guarded_out(M, N, "bf16")
    tg.gemm_bf16(to_dev(A, "bf16"), to_dev(B, "bf16"), C=C)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    check_guard(big, "bf16", M, N, pad)
    return from_dev(C, "bf16")


@pytest.mark.parametrize("shape,rule", [
    ((3, 1000, 700), {"path": "small_m"}),
    ((3, 1000, 700), {"path": "cuda_core", "ctas": 37}),
    ((16, 2048, 4096), {"path": "small_m", "ctas": 74}),
    ((16, 2048, 1000), {"path": "cta_pair"}),
    ((100, 777, 1200), {"path": "one_cta", "ctas": 5}),
    ((300, 520, 640), {"path": "one_cta", "group_m": 3, "ctas": 7}),
    ((300, 520, 640), {"path": "cta_pair", "stages": 4, "group_m": 1, "ctas": 3}),
])
def test_forced_bf16_paths(tg, shape, rule):
    M, N, K = shape
    A, B = synth.normal(M, N, K, seed=3, dtype="bf16", scale_by_sqrt_k=True)
    tg.tune_set([dict({"op": "bf16", "m_lo": M, "m_hi": M}, **rule)])
    got = decode16(_bf16(tg, A, B), "bf16")
    ref = oracle.gemm_bf16(A, B)
    assert_close(got, ref, 1e-2, 1e-2, f"{shape} {rule}")
    assert rel_frob(got, ref) <= 1e-2


def test_reordering_rules_are_bit_identical(tg):
    # 8 x 8 pair tiles for 74 pairs; band height, ring depth and pair count
    # change only which CTA computes a tile and when
    M = N = 2048
    A, B = synth.normal(M, N, 512, seed=2, dtype="bf16", scale_by_sqrt_k=True)
    first = _bf16(tg, A, B)
    for rule in ({"group_m": 1}, {"group_m": 3, "ctas": 11}, {"stages": 4, "group_m": 16},
                 {"path": "cta_pair", "stages": 4, "ctas": 64}):
        tg.tune_set([dict({"op": "bf16", "m_lo": 129}, **rule)])
        assert np.array_equal(_bf16(tg, A, B), first), rule


def test_forced_4bit_paths(tg):
    import torch
    for M, rule in ((2, {"path": "small_m", "ctas": 60}), (16, {"path": "cta_pair"}),
                    (300, {"path": "one_cta", "group_m": 2}), (3, {"path": "cuda_core", "ctas": 9})):
        A, Bq, S, _ = synth.w4a16(M, 1000, 512, seed=4)
        tg.tune_set([dict({"op": "w4a16", "m_lo": M, "m_hi": M}, **rule)])
        C = tg.gemm_w4a16(to_dev(A, "f16"), to_dev(Bq, "u8"), to_dev(S, "f16"), 1000)
        torch.cuda.synchronize()
        assert tg.last_device_status() == 0
        assert_close(decode16(from_dev(C, "f16"), "f16"), oracle.gemm_w4a16(A, Bq, S, N=1000),
                     1e-2, 1e-2, f"w4a16 {M} {rule}")
    for M, rule in ((16, {"path": "cta_pair", "ctas": 5}), (300, {"path": "one_cta"}),
                    (300, {"path": "cta_pair", "group_m": 1})):
        A, Bq, E, _ = synth.wfp4(M, 1000, 480, seed=4)
        tg.tune_set([dict({"op": "wfp4", "m_lo": M, "m_hi": M}, **rule)])
        C = tg.gemm_wfp4(to_dev(A, "bf16"), to_dev(Bq, "u8"), to_dev(E, "u8"), 1000)
        torch.cuda.synchronize()
        assert tg.last_device_status() == 0
        assert_close(decode16(from_dev(C, "bf16"), "bf16"), oracle.gemm_wfp4(A, Bq, E, N=1000),
                     1e-2, 1e-2, f"wfp4 {M} {rule}")


@pytest.mark.parametrize("splits", [1, 3, 8])
def test_forced_ffma_splits(tg, splits):
    import torch
    M, N, K = 200, 200, 1000              # 8 k-slices of 128 -> 8 ranges at most
    A, B = synth.integers(M, N, K, seed=1)
    tg.tune_set([{"op": "f32_ffma", "splits": splits}])
    C = tg.gemm_f32(to_dev(A, "f32"), to_dev(B, "f32"))
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    assert np.array_equal(from_dev(C, "f32"), oracle.round_f32(oracle.gemm_f32(A, B)))


def test_forced_tf32_launch_shape(tg):
    import torch
    A, B = synth.normal(640, 1000, 300, seed=1)
    tg.tune_set([{"op": "f32_tf32", "group_m": 1, "ctas": 6}])
    C = tg.gemm_f32(to_dev(A, "f32"), to_dev(B, "f32"), mode=tg.F32_TF32)
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    assert rel_frob(from_dev(C, "f32"), oracle.gemm_f32(A, B)) <= 5e-3
