"""Host checks of bench.py's measurement arithmetic (no GPU needed).

The roofline fraction of every bench line is achieved / peak, and achieved
is the algorithmic flops or bytes of one launch over its time.  These tests
pin those per-launch counts and each workload's bound to the figures worked
out by hand for the configurations (flops = 2*M*N*K; bytes = operands read
once plus C written once, packed 4-bit weights at half a byte), and check
that the committed DRAM-traffic record is only used for the kernel sources
it was measured on.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

# measured-peak stand-ins with the pool's ridge (~257 flop/byte)
PEAKS = {"hbm_gbs": 6549.0, "bf16_tflops": 1686.0, "bf16_tflops_sustained": 1395.0,
         "sm_max_mhz": 1965.0}

# workload -> (GFLOP, MB of algorithmic traffic, bound), hand-computed
EXPECTED = {
    "bf16_gemm_8192": (1099.5, 402.7, "tensor"),
    "bf16_gemm_8192_relu": (1099.5, 402.7, "tensor"),
    "f16_gemm_8192": (1099.5, 402.7, "tensor"),
    "bf16_gemm_4096": (137.4, 100.7, "tensor"),
    "f16_gemm_4096_relu": (137.4, 100.7, "tensor"),
    "f32_ffma_gemm_4096": (137.4, 201.3, "alu"),
    "f32_ffma_gemm_1024": (2.147, 12.58, "alu"),
    "f32_tf32_gemm_4096": (137.4, 201.3, "tensor"),
    "bf16_gemm_16x8192x8192": (2.147, 134.7, "hbm"),
    "bf16_gemm_128x14336x4096": (15.03, 122.2, "hbm"),
    "bf16_gemm_8192x1024x8192": (137.4, 167.8, "tensor"),
    "bf16_gemm_3000x5000x4000": (120.0, 94.0, "tensor"),
    "w4a16_gemm_m1": (0.1342, 34.62, "hbm"),
    "w4a16_gemm_m16": (2.147, 35.13, "hbm"),
    "w4a16_gemm_m4096": (549.8, 168.8, "tensor"),
    # FP4 weights: 33.55 MB codes + 2.10 MB E8M0 bytes (one per 32 k per column)
    "wfp4_gemm_m1": (0.1342, 35.68, "hbm"),
    "wfp4_gemm_m16": (2.147, 36.18, "hbm"),
    "wfp4_gemm_m4096": (549.8, 169.9, "tensor"),
    # 2:4 sparse A: M*N*K flops (kept values only); Ac 67.1 MB + codes 8.4 MB
    # + B 134.2 MB + C 134.2 MB
    "sp24_bf16_gemm_8192": (549.8, 343.9, "tensor"),
}


def test_every_workload_has_expected_figures():
    assert set(bench.WORKLOADS) == set(EXPECTED)


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_workload_facts(name):
    gflop, mb, bound = EXPECTED[name]
    flops, alg_bytes, got_bound, peak, unit = bench.workload_facts(name, PEAKS)
    assert flops / 1e9 == pytest.approx(gflop, rel=2e-3)
    assert alg_bytes / 1e6 == pytest.approx(mb, rel=2e-3)
    assert got_bound == bound
    if bound == "hbm":
        assert (peak, unit) == (PEAKS["hbm_gbs"], "GB/s")
    elif bound == "alu":
        assert unit == "TFLOP/s" and peak == pytest.approx(148 * 128 * 2 * 1965e6 / 1e12)
    else:
        ratio = 1.1 / 2.25 if name.startswith("f32_tf32") else 1.0
        assert (peak, unit) == (pytest.approx(PEAKS["bf16_tflops"] * ratio), "TFLOP/s")


@pytest.mark.parametrize("name", sorted(bench.TRANSPOSED))
def test_transposed_variants_count_as_their_workload(name):
    base = bench.TRANSPOSED[name][0]
    assert bench.workload_facts(name, PEAKS) == bench.workload_facts(base, PEAKS)


def test_packed_weight_bytes_match_the_generator():
    """The 4-bit byte count equals the arrays the generator produces."""
    host = bench.make_inputs("w4a16_gemm_m1")
    kind, M, N, K = bench.WORKLOADS["w4a16_gemm_m1"][:4]
    nbytes = host["A"].nbytes + host["Bq"].nbytes + host["S"].nbytes + M * N * 2
    assert bench.workload_facts("w4a16_gemm_m1", PEAKS)[1] == nbytes


def test_fp4_weight_bytes_match_the_generator():
    host = bench.make_inputs("wfp4_gemm_m16")
    kind, M, N, K = bench.WORKLOADS["wfp4_gemm_m16"][:4]
    nbytes = host["A"].nbytes + host["Bq"].nbytes + host["S"].nbytes + M * N * 2
    assert bench.workload_facts("wfp4_gemm_m16", PEAKS)[1] == nbytes


def test_traffic_record_follows_the_source_digest(monkeypatch):
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    key, digest, nbytes = next(r for r in rows if r[0] == "bf16_gemm_8192")
    monkeypatch.setattr(bench, "source_digest", lambda files=None: digest)
    assert bench.traffic_record("bf16_gemm_8192") == float(nbytes)
    monkeypatch.setattr(bench, "source_digest", lambda files=None: "0" * 12)
    assert bench.traffic_record("bf16_gemm_8192") is None


def test_headline_sources_exist():
    csrc = os.path.join(ROOT, "tiled_dense_gemm_tma_b200", "csrc")
    for f in bench.HEADLINE_SOURCES:
        assert os.path.exists(os.path.join(csrc, f)), f


def test_sweep_pick_needs_a_margin():
    # candidate 0 is the default; a faster candidate wins only by more than 2 %
    assert bench.sweep_pick([[1.0, 2.0], [0.99, 1.98]]) == 0
    assert bench.sweep_pick([[1.0, 2.0], [0.99, 1.98], [0.5, 3.0]]) == 2
    assert bench.sweep_pick([[1.0], [0.97]]) == 1


def test_sweep_candidates_are_valid_rules():
    """Every candidate the sweep can install is accepted by the library
    (checked on the host: tg_tune_set validates without a device)."""
    from tiled_dense_gemm_tma_b200 import binding as b, build as tg_build
    tg_build.build()
    try:
        for op, m_lo, m_hi, n_lo, n_hi, wls, cands in bench.SWEEP_CLASSES:
            for w in wls:
                kind, M, N = bench.WORKLOADS[w][:3]
                assert m_lo <= M <= m_hi and n_lo <= N <= n_hi, (op, w)
            for cand in cands:
                b.tune_set([dict({"op": op, "m_lo": m_lo, "m_hi": m_hi, "n_lo": n_lo,
                                  "n_hi": n_hi}, **cand)])
    finally:
        b.tune_set([])


def test_generated_tune_table_compiles(tmp_path):
    """The sweep's C++ output compiles against tune.h and its rules read back."""
    import shutil
    import subprocess
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    rules = [{"op": 0, "path": 2, "m_lo": 5, "m_hi": 64, "n_lo": 1, "n_hi": bench.INF,
              "ctas": 112, "group_m": 0, "splits": 0, "stages": 0},
             {"op": 4, "path": 0, "m_lo": 1, "m_hi": 1024, "n_lo": 1, "n_hi": 1024,
              "ctas": 0, "group_m": 0, "splits": 3, "stages": 0}]
    (tmp_path / "tune_table.h").write_text(bench.tune_table_source(rules, ["a", "b"]))
    (tmp_path / "main.cpp").write_text(
        '#include <cstdio>\n#include "tune_table.h"\n'
        'int main() { for (const auto& r : tg::kBuiltinRules) std::printf("%d %d %lld %lld %d %d\\n",'
        ' r.op, r.path, (long long)r.m_lo, (long long)r.n_hi, r.ctas, r.splits); }\n')
    csrc = os.path.join(ROOT, "tiled_dense_gemm_tma_b200", "csrc")
    exe = tmp_path / "t"
    subprocess.run([gxx, "-std=c++17", "-I", str(tmp_path), "-I", csrc, str(tmp_path / "main.cpp"),
                    "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    assert out[0] == f"0 2 5 {bench.INF} 112 0"
    assert out[1] == "4 0 1 1024 0 3"
    assert out[2].startswith("-1 ")
