"""Write synth_sha256.txt: SHA-256 digests of the seeded inputs the parity
tests draw, so that any change to the generator (a draw order, a rounding, a
distribution, a numpy stream change) shows up as a failing test instead of
silently changing every test's inputs.

Calls only the generator (tiled_dense_gemm_tma_b200.synth); the digests
pin inputs, not results.  Run from the repository root:

    python tests/golden/make_synth_sha256.py
"""
import hashlib
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from tiled_dense_gemm_tma_b200 import synth  # noqa: E402

# name -> a call of the generator with the arguments the tests use
CASES = {
    "uniform_pm1_f32_256_seed0": lambda: synth.uniform_pm1(256, 256, 256, 0),
    "normal_f32_1024_seed1": lambda: synth.normal(1024, 1024, 1024, 1),
    "integers_f32_1024_seed1": lambda: synth.integers(1024, 1024, 1024, 1),
    "normal_bf16_300x520x200_seed2_sqrtk": lambda: synth.normal(300, 520, 200, 2, "bf16", True),
    "normal_f16_300x520x200_seed2_sqrtk": lambda: synth.normal(300, 520, 200, 2, "f16", True),
    "integers_bf16_200x300x256_seed1_pm1": lambda: synth.integers(200, 300, 256, 1, lo=-1, hi=1,
                                                                   dtype="bf16"),
    "normal_bf16_128x14336x4096_seed3_sqrtk": lambda: synth.normal(128, 14336, 4096, 3, "bf16", True),
    "w4a16_16x8192x8192_seed4": lambda: synth.w4a16(16, 8192, 8192, 4),
    "w4a16_130x300x384_seed4": lambda: synth.w4a16(130, 300, 384, 4),
    "wfp4_16x8192x8192_seed4": lambda: synth.wfp4(16, 8192, 8192, 4),
    "wfp4_130x300x384_seed4": lambda: synth.wfp4(130, 300, 384, 4),
    "sp24_bf16_300x520x640_seed2": lambda: synth.sp24(300, 520, 640, 2, "bf16"),
    "sp24_f16_16x4096x4096_seed3": lambda: synth.sp24(16, 4096, 4096, 3, "f16"),
}


def digest(arrays):
    h = hashlib.sha256()
    for a in arrays:
        a = np.ascontiguousarray(a)
        h.update(f"{a.dtype.str}{a.shape}".encode())
        h.update(a.tobytes())
    return h.hexdigest()


def compute():
    return {name: digest(fn()) for name, fn in CASES.items()}


if __name__ == "__main__":
    with open(os.path.join(HERE, "synth_sha256.txt"), "w") as f:
        f.write("# SHA-256 of the seeded inputs (dtype, shape and bytes of each array the\n")
        f.write("# generator returns, in order); written by make_synth_sha256.py\n")
        for name, d in compute().items():
            f.write(f"{name} {d}\n")
