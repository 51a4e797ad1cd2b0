"""The seeded input generator: determinism, distributions and packing."""
import hashlib

import numpy as np

from tiled_dense_gemm_tma_b200 import synth


def _h(*arrays):
    h = hashlib.sha256()
    for a in arrays:
        h.update(np.ascontiguousarray(a).tobytes())
    return h.hexdigest()


def test_same_seed_same_bytes():
    assert _h(*synth.normal(33, 17, 65, 2, "bf16", True)) == _h(*synth.normal(33, 17, 65, 2, "bf16", True))
    assert _h(*synth.uniform_pm1(8, 9, 10, 0)) == _h(*synth.uniform_pm1(8, 9, 10, 0))
    assert _h(*synth.w4a16(2, 16, 256, 4)) == _h(*synth.w4a16(2, 16, 256, 4))
    assert _h(*synth.normal(8, 9, 10, 1)) != _h(*synth.normal(8, 9, 10, 2))


def test_distributions():
    A, B = synth.uniform_pm1(256, 256, 256, 0)
    assert A.dtype == np.float32 and A.min() >= -1 and A.max() <= 1
    assert abs(A.mean()) < 0.01 and abs(A.var() - 1 / 3) < 0.01
    A, B = synth.normal(512, 512, 1024, 2, "f16", True)
    a = A.view(np.float16).astype(np.float64)
    assert abs(a.std() * np.sqrt(1024) - 1) < 0.02
    A, B = synth.integers(64, 64, 64, 1)
    assert set(np.unique(A)) <= set(range(-3, 4)) and len(np.unique(A)) == 7
    A, Bq, s, q = synth.w4a16(4, 64, 512, 4)
    assert Bq.shape == (512, 32) and s.shape == (4, 64) and q.min() == -8 and q.max() == 7
    sv = s.view(np.float16).astype(np.float64)
    assert sv.min() >= 0.005 - 1e-5 and sv.max() <= 0.02 + 1e-5


def test_pack_int4_roundtrip_all_values():
    q = np.array([list(range(-8, 8)) * 2], np.int64)          # 1 x 32
    packed = synth.pack_int4(q)
    lo = (packed & 0xF).astype(np.int64)
    hi = (packed >> 4).astype(np.int64)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    back = np.empty_like(q)
    back[:, 0::2], back[:, 1::2] = lo, hi
    assert np.array_equal(back, q)
    # odd N pads the last high nibble with zero
    assert synth.pack_int4(np.array([[1, 2, 3]])).tolist() == [[0x21, 0x03]]


def test_bf16_store_is_rne_of_fp32():
    x = np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, -2.0, 0.0])
    assert synth.store(x, "bf16").tolist() == [0x3F80, 0x3F80, 0x3F82, 0xC000, 0x0000]


def test_inputs_match_recorded_digests():
    """The generator still draws exactly the recorded inputs (digests in
    tests/golden/synth_sha256.txt, written by make_synth_sha256.py)."""
    import importlib.util
    import os
    golden = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    spec = importlib.util.spec_from_file_location(
        "make_synth_sha256", os.path.join(golden, "make_synth_sha256.py"))
    mk = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mk)
    recorded = {}
    with open(os.path.join(golden, "synth_sha256.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, d = line.split()
                recorded[name] = d
    assert recorded.keys() == mk.CASES.keys()
    assert mk.compute() == recorded


def test_pack_nibbles_roundtrip_all_codes():
    codes = np.arange(16, dtype=np.uint8).reshape(2, 8)
    packed = synth.pack_nibbles(codes)
    assert packed.shape == (2, 4)
    lo, hi = packed & 0xF, packed >> 4
    assert np.array_equal(lo, codes[:, 0::2]) and np.array_equal(hi, codes[:, 1::2])
    odd = synth.pack_nibbles(codes[:, :7])          # odd N: zero padding nibble
    assert odd.shape == (2, 4) and np.all(odd[:, 3] >> 4 == 0)


def test_wfp4_inputs():
    A, Bq, E, codes = synth.wfp4(3, 70, 96, seed=4)
    assert A.dtype == np.uint16 and A.shape == (3, 96)
    assert Bq.shape == (96, 35) and E.shape == (3, 70) and codes.shape == (96, 70)
    assert E.dtype == np.uint8 and E.min() >= 118 and E.max() <= 122
    assert set(np.unique(codes)) == set(range(16))
    assert np.array_equal(Bq, synth.pack_nibbles(codes))
