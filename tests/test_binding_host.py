"""Host checks of the Python binding's marshalling (no GPU needed).

The binding turns torch tensors into the C ABI's pointers, leading
dimensions and transpose flags, and builds the differentiable matmul from
those calls.  Here the library is replaced by a fake that reads its operands
back through exactly those pointers and pitches (CPU tensors, so the
addresses are host memory) and multiplies them in float64.  A wrong pitch,
flag or operand order then gives a wrong product, and the forward and
backward results are compared with torch's own CPU matmul.
"""
import ctypes

import numpy as np
import pytest
import torch

from tiled_dense_gemm_tma_b200 import binding


def _read(ptr, rows, cols, ld):
    """rows x cols bf16 matrix at host address ptr, row pitch ld elements."""
    if rows == 0 or cols == 0:
        return np.zeros((rows, cols))
    n = (rows - 1) * ld + cols
    raw = np.ctypeslib.as_array((ctypes.c_uint16 * n).from_address(ptr))
    u = np.empty(rows * ld, np.uint16)
    u[:n] = raw
    bits = u.reshape(rows, ld)[:, :cols].astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def _write(ptr, M, N, ld, val):
    out = torch.from_numpy(val.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    for i in range(M):
        row = np.ctypeslib.as_array((ctypes.c_int16 * N).from_address(ptr + 2 * i * ld))
        row[:] = out[i]


class FakeLib:
    """Records every call and computes C = op(A) op(B) from raw memory."""

    def __init__(self):
        self.calls = []

    def tg_gemm_bf16(self, M, N, K, A, lda, B, ldb, C, ldc, epi, stream):
        return self.tg_gemm_bf16_ex(M, N, K, A, lda, 0, B, ldb, 0, C, ldc, epi, stream, "plain")

    def tg_gemm_bf16_ex(self, M, N, K, A, lda, ta, B, ldb, tb, C, ldc, epi, stream, kind="ex"):
        self.calls.append(dict(kind=kind, M=M, N=N, K=K, A=A, lda=lda, ta=ta, B=B, ldb=ldb,
                               tb=tb, C=C, ldc=ldc))
        a = _read(A, K, M, lda).T if ta else _read(A, M, K, lda)
        b = _read(B, N, K, ldb).T if tb else _read(B, K, N, ldb)
        c = a @ b
        if epi == 1:
            c = np.maximum(c, 0)
        _write(C, M, N, ldc, c)
        return 0


def _read_bytes(ptr, rows, cols, ld, dtype):
    """rows x cols array of `dtype` at host address ptr, row pitch ld elements."""
    if rows == 0 or cols == 0:
        return np.zeros((rows, cols), dtype)
    ct = ctypes.c_uint16 if dtype == np.uint16 else ctypes.c_uint8
    n = (rows - 1) * ld + cols
    raw = np.ctypeslib.as_array((ct * n).from_address(ptr)).astype(dtype)
    u = np.zeros(rows * ld, dtype)
    u[:n] = raw
    return np.ascontiguousarray(u.reshape(rows, ld)[:, :cols])


def _fake_wfp4(self, M, N, K, A, lda, Bq, ldbq, S, lds, block, C, ldc, epi, stream):
    """Reads the FP4-weight operands back through the pointers and pitches it
    is given and multiplies them with the oracle."""
    import oracle
    self.calls.append(dict(kind="wfp4", M=M, N=N, K=K, lda=lda, ldbq=ldbq, lds=lds, block=block))
    a = _read_bytes(A, M, K, lda, np.uint16)
    q = _read_bytes(Bq, K, (N + 1) // 2, ldbq, np.uint8)
    e = _read_bytes(S, (K + block - 1) // block, N, lds, np.uint8)
    _write(C, M, N, ldc, oracle.gemm_wfp4(a, q, e, N=N, block=block, relu=epi == 1))
    return 0


FakeLib.tg_gemm_wfp4 = _fake_wfp4


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(binding, "load_library", lambda: lib)
    monkeypatch.setattr(binding, "_require_cuda", lambda device, *named: None)
    monkeypatch.setattr(binding, "_stream_handle", lambda stream: ctypes.c_void_p(0))
    monkeypatch.setattr(binding, "empty_out",
                        lambda M, N, dtype, device: torch.empty((M, N), dtype=dtype))
    return lib


def _bf16(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(rows, cols, generator=g).to(torch.bfloat16)


def _close(got, ref):
    ref = ref.double()
    err = (got.double() - ref).abs().max().item()
    assert err <= 1e-2 * (1 + ref.abs().max().item()), err


def test_stored_reading_of_views():
    W = torch.empty(24, 40, dtype=torch.bfloat16)          # out x in, row-major
    st, tr = binding._stored(W.t())
    assert tr and st.data_ptr() == W.data_ptr() and tuple(st.shape) == (24, 40)
    st, tr = binding._stored(W)
    assert not tr and st is W
    # a column slice keeps its row pitch: still no copy
    st, tr = binding._stored(W[:, 8:32])
    assert not tr and st.stride(0) == 40
    # (M x 1) transposed view of a (1 x M) row: the aligned reading wins
    r = torch.empty(1, 64, dtype=torch.bfloat16)
    st, tr = binding._stored(r.t())
    assert tr and st.data_ptr() == r.data_ptr()
    # neither reading: copied
    x = torch.empty(16, 32, dtype=torch.bfloat16)[::2, ::2]
    st, tr = binding._stored(x)
    assert not tr and st.is_contiguous() and st.data_ptr() != x.data_ptr()


@pytest.mark.parametrize("ta", [False, True])
@pytest.mark.parametrize("tb", [False, True])
def test_matmul_forward_and_backward_marshalling(fake, ta, tb):
    M, N, K = 24, 40, 32
    A0 = (_bf16(K, M, 1).t() if ta else _bf16(M, K, 1))      # logical M x K
    B0 = (_bf16(N, K, 2).t() if tb else _bf16(K, N, 2))      # logical K x N
    A = A0.detach().requires_grad_(True)
    B = B0.detach().requires_grad_(True)
    C = binding.matmul(A, B)
    fwd = fake.calls[-1]
    assert fwd["kind"] == ("ex" if (ta or tb) else "plain")
    assert (fwd["ta"], fwd["tb"]) == (int(ta), int(tb))
    # the kernels read the caller's storage, not a copy
    assert fwd["A"] == A0.data_ptr() and fwd["B"] == B0.data_ptr()
    _close(C, A0.double() @ B0.double())

    G = _bf16(N, M, 3).t()                                   # a transposed gradient view
    C.backward(G)
    # dA = G B^T, dB = A^T G, computed from the same stored values
    _close(A.grad, G.double() @ B0.double().t())
    _close(B.grad, A0.double().t() @ G.double())
    assert A.grad.shape == A.shape and B.grad.shape == B.shape
    for call in fake.calls[-2:]:
        assert call["kind"] == "ex"          # every backward product reads a transpose


def test_gemm_relu_and_explicit_flags(fake):
    M, N, K = 16, 24, 32
    At = _bf16(K, M, 4)
    Bt = _bf16(N, K, 5)
    C = binding.gemm_bf16(At, Bt, relu=True, trans_a=True, trans_b=True)
    _close(C, (At.double().t() @ Bt.double().t()).clamp_min(0))
    call = fake.calls[-1]
    assert (call["M"], call["N"], call["K"]) == (M, N, K)
    assert (call["lda"], call["ldb"]) == (M, K)


def test_operands_must_be_cuda_tensors():
    A = torch.zeros(8, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        binding.gemm_bf16(A, A)
    with pytest.raises(ValueError, match="2-D"):
        binding.gemm_bf16(A[0], A)
    q = torch.zeros(128, 8, dtype=torch.uint8)
    s = torch.zeros(1, 16, dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA"):
        binding.gemm_w4a16(torch.zeros(4, 128, dtype=torch.float16), q, s, 16)


def test_wfp4_marshalling(fake):
    """gemm_wfp4 passes the activations, packed codes and scale bytes with
    their own pitches (elements for A, bytes for the packed codes and the
    E8M0 rows) and the block size; a wider-than-needed pitch on each operand
    makes a mix-up visible."""
    import oracle
    from tiled_dense_gemm_tma_b200 import synth
    M, N, K = 5, 40, 96
    A, Bq, E, _ = synth.wfp4(M, N, K, seed=3)
    tA = torch.zeros((M, K + 8), dtype=torch.int16)
    tA[:, :K] = torch.from_numpy(A.view(np.int16))
    tA = tA.view(torch.bfloat16)[:, :K]
    tq = torch.zeros((K, 48), dtype=torch.uint8)
    tq[:, :Bq.shape[1]] = torch.from_numpy(Bq)
    te = torch.zeros((E.shape[0], 64), dtype=torch.uint8)
    te[:, :N] = torch.from_numpy(E)
    te = te[:, :N]
    C = binding.gemm_wfp4(tA, tq, te, N, relu=True)
    call = fake.calls[-1]
    assert (call["M"], call["N"], call["K"], call["block"]) == (M, N, K, 32)
    assert (call["lda"], call["ldbq"], call["lds"]) == (K + 8, 48, 64)
    ref = oracle.gemm_wfp4(A, Bq, E, N=N, relu=True)
    _close(C, torch.from_numpy(ref))
    with pytest.raises(TypeError):
        binding.gemm_wfp4(tA.view(torch.float16), tq, te, N)
