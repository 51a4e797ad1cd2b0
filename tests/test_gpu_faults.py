"""Failure detection on the GPU without a fault, for every kernel family: a
wait that can never complete must end with TG_ERR_TIMEOUT, leave the CUDA
context usable, and leave the library able to run the next call correctly.

TG_INJECT=1 makes the first kernel launch of the process (only that one) have
the TMA producer of CTA 0 (of CTA pair 0's leader) skip arming its first
ring slot: a barrier that nothing then completes.  TG_DEBUG_TIMEOUT_US=200000
bounds every barrier wait at 0.2 s.  That CTA gives up, records the timeout
in the device status word, drains its in-flight copies, frees its tensor
memory and exits; the other CTAs finish their work.  In the kernels that
split K across CTAs through global memory (weight-streaming small-M and
CUDA-core M <= 4 under stream-K, fp32 FFMA split-K) the tiles CTA 0
contributes to are then left with incomplete tickets, so the status read
must mark the split-K workspace for re-zeroing (inside a cluster, CTA 0's
peers time out on the partials it never sends and exit with it):
the second call of the same shape on the same stream must match the fp64
oracle.  Each family runs in a child process because both knobs are read once
per process; the one-CTA fallback kernels run with TG_NO_PAIR=1 as well.
"""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys, time, torch
    import numpy as np
    sys.path.insert(0, %r); sys.path.insert(0, %r)
    import oracle
    import tiled_dense_gemm_tma_b200 as tg
    from tiled_dense_gemm_tma_b200 import synth
    from gpu_util import to_dev, from_dev, decode16, assert_close, rel_frob

    fam = sys.argv[1]
    def case():
        # returns (call, check): call() launches once, check(result) compares with the oracle
        if fam in ("tc2_bf16", "tc_bf16", "skinny_bf16", "gemv_bf16", "skinny_bf16_tb"):
            M, N, K = {"tc2_bf16": (512, 768, 512), "tc_bf16": (512, 768, 512),
                       "skinny_bf16": (16, 2048, 4096), "gemv_bf16": (1, 2048, 8192),
                       "skinny_bf16_tb": (16, 2048, 4096)}[fam]
            A, B = synth.normal(M, N, K, seed=2, dtype="bf16", scale_by_sqrt_k=True)
            tb = fam.endswith("_tb")
            dA, dB = to_dev(A, "bf16"), to_dev(np.ascontiguousarray(B.T) if tb else B, "bf16")
            ref = oracle.gemm_bf16(A, B)
            call = lambda: tg.gemm_bf16(dA, dB, trans_b=tb)
            conv = lambda C: decode16(from_dev(C, "bf16"), "bf16")
            tol = (1e-2, 1e-2)
        elif fam in ("ffma", "ffma_splitk", "tf32", "tf32_one"):
            M, N, K = {"ffma": (2048, 1024, 256), "ffma_splitk": (200, 200, 3000),
                       "tf32": (512, 768, 512), "tf32_one": (512, 768, 512)}[fam]
            A, B = synth.normal(M, N, K, seed=1)
            dA, dB = to_dev(A, "f32"), to_dev(B, "f32")
            ref = oracle.gemm_f32(A, B)
            mode = tg.F32_TF32 if fam.startswith("tf32") else tg.F32_FFMA
            call = lambda: tg.gemm_f32(dA, dB, mode=mode)
            conv = lambda C: from_dev(C, "f32")
            tol = None
        elif fam.startswith("w4a16") or fam.startswith("skinny_w4a16") or fam.startswith("gemv_w4a16"):
            M, N, K = {"w4a16_pair": (512, 1024, 1024), "w4a16_large": (512, 1024, 1024),
                       "skinny_w4a16": (16, 2048, 4096), "gemv_w4a16": (2, 2048, 8192),
                       "gemv_w4a16_cluster": (1, 8192, 8192),
                       "skinny_w4a16_cluster": (16, 8192, 4096)}[fam]
            A, Bq, S, _ = synth.w4a16(M, N, K, seed=4)
            dA, dB, dS = to_dev(A, "f16"), to_dev(Bq, "u8"), to_dev(S, "f16")
            ref = oracle.gemm_w4a16(A, Bq, S, N=N)
            call = lambda: tg.gemm_w4a16(dA, dB, dS, N)
            conv = lambda C: decode16(from_dev(C, "f16"), "f16")
            tol = (1e-2, 1e-2)
        elif fam.startswith("sp24"):
            Ac, E, B, _ = synth.sp24(512, 768, 1024, seed=2, dtype="bf16")
            dA, dE, dB = to_dev(Ac, "bf16"), to_dev(E, "u8"), to_dev(B, "bf16")
            ref = oracle.gemm_sp24(Ac, E, B, "bf16")
            call = lambda: tg.gemm_sp24(dA, dE, dB)
            conv = lambda C: decode16(from_dev(C, "bf16"), "bf16")
            tol = (1e-2, 1e-2)
        else:
            M, N, K = {"wfp4_pair": (512, 1024, 1024), "wfp4_large": (512, 1024, 1024),
                       "skinny_wfp4": (16, 2048, 4096), "gemv_wfp4": (3, 2048, 4096),
                       "gemv_wfp4_cluster": (2, 8192, 1024)}[fam]
            A, Bq, E, _ = synth.wfp4(M, N, K, seed=4)
            dA, dB, dE = to_dev(A, "bf16"), to_dev(Bq, "u8"), to_dev(E, "u8")
            ref = oracle.gemm_wfp4(A, Bq, E, N=N)
            call = lambda: tg.gemm_wfp4(dA, dB, dE, N)
            conv = lambda C: decode16(from_dev(C, "bf16"), "bf16")
            tol = (1e-2, 1e-2)
        def check(C):
            got = conv(C)
            if tol is None:
                assert rel_frob(got, ref) <= (5e-3 if fam.startswith("tf32") else 1e-5), fam
            else:
                assert_close(got, ref, tol[0], tol[1], fam)
        return call, check

    call, check = case()
    torch.cuda.synchronize()
    t0 = time.time()
    call()                                  # the injected launch
    st = tg.last_device_status()
    dt = time.time() - t0
    st2 = tg.last_device_status()
    C = call()                              # a normal launch on the same stream
    st3 = tg.last_device_status()
    check(C)
    x = (torch.ones(1024, device="cuda") * 2).sum().item()
    print("RESULT", st, st2, st3, x, round(dt, 3))
""") % (ROOT, os.path.join(ROOT, "tests"))

# *_cluster: shapes whose split-K runs inside clusters (the owners'
# byte-counting barriers and the closing cluster barrier abort too)
FAMILIES = ["tc2_bf16", "tf32", "skinny_bf16", "skinny_bf16_tb", "gemv_bf16", "ffma",
            "ffma_splitk", "w4a16_pair", "skinny_w4a16", "skinny_w4a16_cluster", "gemv_w4a16",
            "gemv_w4a16_cluster",
            "wfp4_pair", "skinny_wfp4", "gemv_wfp4", "gemv_wfp4_cluster", "sp24_pair", "tc_bf16",
            "w4a16_large", "wfp4_large", "sp24_one", "tf32_one"]
# run with the CTA-pair kernels off
ONE_CTA = {"tc_bf16", "w4a16_large", "wfp4_large", "sp24_one", "tf32_one"}


@pytest.mark.parametrize("family", FAMILIES)
def test_bounded_wait_reports_timeout_then_recovers(family):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, TG_INJECT="1", TG_DEBUG_TIMEOUT_US="200000")
    if family in ONE_CTA:
        env["TG_NO_PAIR"] = "1"
    r = subprocess.run([sys.executable, "-c", CHILD, family], env=env, capture_output=True,
                       text=True, timeout=180)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("RESULT")][0].split()
    st, st2, st3, x, dt = int(line[1]), int(line[2]), int(line[3]), float(line[4]), float(line[5])
    assert st == 5                      # TG_ERR_TIMEOUT from the injected launch
    assert st2 == 0                     # cleared by the first read
    assert st3 == 0                     # the next launch ran normally (and matched the oracle)
    assert x == 2048.0                  # context still usable
    assert dt < 30.0
