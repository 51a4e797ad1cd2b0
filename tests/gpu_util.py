"""Helpers for GPU parity tests: numpy <-> torch marshalling, guard bands,
tolerance checks.  Holds no GEMM arithmetic."""
import numpy as np

SENTINEL16 = 0x7BAD          # an fp16 / bf16 bit pattern never produced by the tests
SENTINEL32 = np.float32(-12345.678)


def to_dev(arr, kind):
    """numpy stored values -> CUDA tensor. kind: 'f32', 'f16', 'bf16', 'u8'.

    The device copy's row pitch is rounded up to a multiple of 16 bytes (the
    library requires it), so odd widths come back as strided views."""
    import torch
    arr = np.asarray(arr)
    rows, cols = arr.shape
    eb = {"f32": 4, "u8": 1}.get(kind, 2)
    per = 16 // eb
    ld = max(per, -(-cols // per) * per)
    if kind == "f32":
        host = np.zeros((rows, ld), np.float32)
        host[:, :cols] = arr
        t = torch.from_numpy(host).cuda()
    elif kind == "u8":
        host = np.zeros((rows, ld), np.uint8)
        host[:, :cols] = arr
        t = torch.from_numpy(host).cuda()
    else:
        host = np.zeros((rows, ld), np.uint16)
        host[:, :cols] = arr
        t = torch.from_numpy(host.view(np.int16)).cuda()
        t = t.view(torch.float16 if kind == "f16" else torch.bfloat16)
    return t[:, :cols]


def from_dev(t, kind):
    """CUDA tensor -> numpy (float32 values, or uint16 bits for f16/bf16)."""
    import torch
    if kind == "f32":
        return t.float().cpu().numpy()
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def decode16(bits, kind):
    b = np.asarray(bits, np.uint16)
    if kind == "f16":
        return b.view(np.float16).astype(np.float64)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def guarded_out(M, N, kind, pad_r=3, pad_c=None):
    """An output view C (M x N) inside a larger buffer whose margin holds a
    sentinel; returns (big, C).  Row pitch is padded too."""
    import torch
    eb = 4 if kind == "f32" else 2
    pc = pad_c if pad_c is not None else 16 // eb
    ld = N + 2 * pc
    ld += (-ld) % (16 // eb)
    if kind == "f32":
        big = torch.full((M + 2 * pad_r, ld), float(SENTINEL32), dtype=torch.float32, device="cuda")
    else:
        dt = torch.float16 if kind == "f16" else torch.bfloat16
        big = torch.full((M + 2 * pad_r, ld), SENTINEL16, dtype=torch.int16, device="cuda").view(dt)
    C = big[pad_r:pad_r + M, pc:pc + N]
    return big, C, (pad_r, pc)


def check_guard(big, kind, M, N, pad):
    """Everything outside the C window must still hold the sentinel."""
    pr, pc = pad
    host = from_dev(big, kind)
    mask = np.ones(host.shape, bool)
    mask[pr:pr + M, pc:pc + N] = False
    if kind == "f32":
        assert np.all(host[mask] == SENTINEL32), "write outside C"
    else:
        assert np.all(host[mask] == SENTINEL16), "write outside C"


def assert_close(got, ref, rtol, atol, what=""):
    """|got - ref| <= atol + rtol * |ref| elementwise (assert_close semantics)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at "
                             f"{tuple(i)} got {got[tuple(i)]} ref {ref[tuple(i)]}")


def rel_frob(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got))
