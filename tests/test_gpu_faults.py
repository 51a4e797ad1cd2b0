"""Failure detection on the GPU without a fault: a wait that can never
complete must end with TG_ERR_TIMEOUT and leave the CUDA context usable.

TG_INJECT=1 makes the tensor-core kernel's producer skip arming its first
ring slot (a flag that nothing then sets); TG_DEBUG_TIMEOUT_US=200000 bounds
every barrier wait at 0.2 s.  Each CTA then gives up, records the timeout in
the device status word, drains its in-flight copies, frees its tensor memory
and exits.  The run happens in a child process because both knobs are read
once per process.
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
    sys.path.insert(0, %r)
    import tiled_dense_gemm_tma_b200 as tg
    A = torch.randn(512, 512, device="cuda", dtype=torch.bfloat16)
    B = torch.randn(512, 512, device="cuda", dtype=torch.bfloat16)
    t0 = time.time()
    tg.gemm_bf16(A, B)
    st = tg.last_device_status()
    dt = time.time() - t0
    # the context must still work: a torch op and another status read
    x = (torch.ones(1024, device="cuda") * 2).sum().item()
    st2 = tg.last_device_status()
    print("RESULT", st, st2, x, round(dt, 3))
""") % ROOT


def test_bounded_wait_reports_timeout():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, TG_INJECT="1", TG_DEBUG_TIMEOUT_US="200000")
    r = subprocess.run([sys.executable, "-c", CHILD], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("RESULT")][0].split()
    st, st2, x, dt = int(line[1]), int(line[2]), float(line[3]), float(line[4])
    assert st == 5                      # TG_ERR_TIMEOUT
    assert st2 == 0                     # cleared by the first read
    assert x == 2048.0                  # context still usable
    assert dt < 30.0
