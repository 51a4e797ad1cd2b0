"""CUDA graph capture of library calls on a stream the library has never
seen, checked against the fp64 oracle after replays.

A call that would need the per-stream split-K workspace cannot allocate it
while the stream is being captured.  The CTA-pair kernel then runs its last
wave of tiles whole instead of split (4096^3: 256 pair tiles on 74 pairs
would split the last 34; 128 x 4096 x 1024, operand-swapped: 16 pair tiles,
all split); the small-M 16-bit GEMM whose split runs inside thread-block
clusters needs no workspace at all.  All must capture, replay and match the
oracle (rtol = atol = 1e-2, relative Frobenius error <= 1e-2 for bf16).
The small-M call takes the same kernel and plan captured or not, so its
replayed result must equal an uncaptured call's bit for bit.  One uncaptured call of each shape on another stream comes first,
so the kernels' one-time set-up (attributes, descriptors) is done outside
the capture, as the header asks.
"""
import numpy as np
import pytest

import oracle
from tiled_dense_gemm_tma_b200 import synth
from gpu_util import to_dev, from_dev, decode16, assert_close, rel_frob

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tg():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import tiled_dense_gemm_tma_b200 as tg
    tg.load_library()
    return tg


@pytest.mark.parametrize("shape", [(4096, 4096, 4096), (16, 8192, 4096), (128, 4096, 1024)])
def test_capture_on_a_fresh_stream(tg, shape):
    import torch
    M, N, K = shape
    same_plan = M <= 64                                      # the weight-streaming kernel
    A, B = synth.normal(M, N, K, seed=21, dtype="bf16", scale_by_sqrt_k=True)
    dA, dB = to_dev(A, "bf16"), to_dev(B, "bf16")
    C0 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    tg.gemm_bf16(dA, dB, C=C0)                               # uncaptured, default stream
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()                                  # never used by the library
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        tg.gemm_bf16(dA, dB, C=C)
    for _ in range(3):
        C.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert tg.last_device_status() == 0
    bits = from_dev(C, "bf16")
    got = decode16(bits, "bf16")
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, min(M, 24), replace=False)]))
    ref = oracle.gemm_bf16(np.ascontiguousarray(A[rows]), B)
    assert_close(got[rows], ref, 1e-2, 1e-2, f"graph {shape}")
    assert rel_frob(got[rows], ref) <= 1e-2
    if same_plan:
        assert np.array_equal(bits, from_dev(C0, "bf16")), "captured vs uncaptured"
    del g
