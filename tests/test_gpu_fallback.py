"""The one-CTA tensor-core kernels are the fallback when a cluster (CTA-pair)
launch is refused.  TG_NO_PAIR=1 makes every pair launch report
"unsupported" (read once per process, so the check runs in a child
process); bf16, fp16, w4a16 and FP4-weight GEMMs with M > 128, and the 2:4
sparse GEMM, must then still match the fp64 oracle at rtol = atol = 1e-2, on
shapes with one tile per CTA and with more tiles than CTAs.
"""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys
    sys.path.insert(0, %r); sys.path.insert(0, %r)
    import torch
    import oracle
    import tiled_dense_gemm_tma_b200 as tg
    from tiled_dense_gemm_tma_b200 import synth
    from gpu_util import to_dev, from_dev, decode16, assert_close
    tg.load_library()
    for kind in ("bf16", "f16"):
        A, B = synth.normal(300, 520, 256, seed=2, dtype=kind, scale_by_sqrt_k=True)
        fn = tg.gemm_bf16 if kind == "bf16" else tg.gemm_f16
        C = fn(to_dev(A, kind), to_dev(B, kind), relu=True)
        ref = (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B, True)
        assert_close(decode16(from_dev(C, kind), kind), ref, 1e-2, 1e-2, kind)
    # 16 x 11 = 176 tiles of 128 x 256 for 148 persistent CTAs: CTAs run a
    # second tile (accumulator double buffer, ring phases across tiles)
    for kind in ("bf16", "f16"):
        A, B = synth.normal(2000, 2600, 320, seed=2, dtype=kind, scale_by_sqrt_k=True)
        fn = tg.gemm_bf16 if kind == "bf16" else tg.gemm_f16
        C = fn(to_dev(A, kind), to_dev(B, kind))
        ref = (oracle.gemm_bf16 if kind == "bf16" else oracle.gemm_f16)(A, B)
        assert_close(decode16(from_dev(C, kind), kind), ref, 1e-2, 1e-2, kind + " many tiles")
    for (M, N, K) in ((257, 520, 384), (2048, 2600, 512)):
        A, Bq, S, _ = synth.w4a16(M, N, K, seed=4)
        C = tg.gemm_w4a16(to_dev(A, "f16"), to_dev(Bq, "u8"), to_dev(S, "f16"), N)
        assert_close(decode16(from_dev(C, "f16"), "f16"), oracle.gemm_w4a16(A, Bq, S, N=N),
                     1e-2, 1e-2, f"w4a16 {M}x{N}x{K}")
    for (M, N, K) in ((257, 520, 384), (2048, 2600, 480)):
        A, Bq, E, _ = synth.wfp4(M, N, K, seed=4)
        C = tg.gemm_wfp4(to_dev(A, "bf16"), to_dev(Bq, "u8"), to_dev(E, "u8"), N)
        assert_close(decode16(from_dev(C, "bf16"), "bf16"), oracle.gemm_wfp4(A, Bq, E, N=N),
                     1e-2, 1e-2, f"wfp4 {M}x{N}x{K}")
    for (M, N, K) in ((300, 520, 200), (2048, 2600, 256)):
        Ac, E, B, _ = synth.sp24(M, N, K, seed=2, dtype="bf16")
        C = tg.gemm_sp24(to_dev(Ac, "bf16"), to_dev(E, "u8"), to_dev(B, "bf16"))
        assert_close(decode16(from_dev(C, "bf16"), "bf16"), oracle.gemm_sp24(Ac, E, B, "bf16"),
                     1e-2, 1e-2, f"sp24 {M}x{N}x{K}")
    torch.cuda.synchronize()
    print("RESULT", tg.last_device_status())
""") % (ROOT, os.path.join(ROOT, "tests"))


def test_one_cta_fallback_kernels():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, TG_NO_PAIR="1")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("RESULT")][0].split()
    assert int(line[1]) == 0
