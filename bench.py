#!/usr/bin/env python3
"""Benchmark of the tiled dense GEMM library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference] [--no-breakdown]
    python bench.py --sweep        (one GPU: rewrite the built-in tuning rules)

A step is one call of the whole hot path for one GEMM of the workload:
argument validation and tensor-map lookup on the host, then the persistent
kernel (tile scheduling, TMA staging ring, tensor-core mainloop, epilogue).
Inputs are seeded synthetic matrices (tiled_dense_gemm_tma_b200.synth),
resident in HBM before timing starts.  The headline workload is the bf16
GEMM M = N = K = 8192 with N(0,1)/sqrt(K) entries; its inputs (256 MB) are
larger than the 126 MB L2, so steps run back to back without an L2 flush.
The per-dtype breakdown flushes L2 before every timed launch (writes one
512 MB buffer, then reads another, so no dirty lines are left to write back
during the timed launch).

Prints ONE JSON line on rank 0.  With --impl reference it times the CPU
oracle (fp64 triple loop) on a bounded sample of the same workload instead.
"""
import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from tiled_dense_gemm_tma_b200 import synth  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 512 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
N_SMS_B200 = 148
FFMA_LANES_PER_SM = 128


# --------------------------------------------------------------- workloads

WORKLOADS = {
    # name: kind, M, N, K, seed, relu, distribution
    "bf16_gemm_8192": ("bf16", 8192, 8192, 8192, 2, False, "normal_sqrtk"),
    "bf16_gemm_8192_relu": ("bf16", 8192, 8192, 8192, 2, True, "normal_sqrtk"),
    "f16_gemm_8192": ("f16", 8192, 8192, 8192, 2, False, "normal_sqrtk"),
    "bf16_gemm_4096": ("bf16", 4096, 4096, 4096, 2, False, "normal_sqrtk"),
    "f16_gemm_4096_relu": ("f16", 4096, 4096, 4096, 2, True, "normal_sqrtk"),
    "f32_ffma_gemm_4096": ("f32_ffma", 4096, 4096, 4096, 1, False, "normal"),
    "f32_ffma_gemm_1024": ("f32_ffma", 1024, 1024, 1024, 1, False, "normal"),
    "f32_tf32_gemm_4096": ("f32_tf32", 4096, 4096, 4096, 1, False, "normal"),
    "bf16_gemm_16x8192x8192": ("bf16", 16, 8192, 8192, 3, False, "normal_sqrtk"),
    "bf16_gemm_128x14336x4096": ("bf16", 128, 14336, 4096, 3, False, "normal_sqrtk"),
    "bf16_gemm_8192x1024x8192": ("bf16", 8192, 1024, 8192, 3, False, "normal_sqrtk"),
    "bf16_gemm_3000x5000x4000": ("bf16", 3000, 5000, 4000, 3, False, "normal_sqrtk"),
    "w4a16_gemm_m1": ("w4a16", 1, 8192, 8192, 4, False, "w4a16"),
    "w4a16_gemm_m16": ("w4a16", 16, 8192, 8192, 4, False, "w4a16"),
    "w4a16_gemm_m4096": ("w4a16", 4096, 8192, 8192, 4, False, "w4a16"),
    # FP4-weight GEMM: bf16 A N(0,1), E2M1 codes uniform over all 16, E8M0
    # block exponents uniform in {118..122}, the 4-bit workload's shapes
    "wfp4_gemm_m1": ("wfp4", 1, 8192, 8192, 4, False, "wfp4"),
    "wfp4_gemm_m16": ("wfp4", 16, 8192, 8192, 4, False, "wfp4"),
    "wfp4_gemm_m4096": ("wfp4", 4096, 8192, 8192, 4, False, "wfp4"),
    # 2:4 structured-sparse A (two kept values per chunk of 4 k, N(0,1)/sqrt(K/2);
    # the six position pairs uniform), dense B N(0,1)/sqrt(K)
    "sp24_bf16_gemm_8192": ("sp24_bf16", 8192, 8192, 8192, 2, False, "sp24"),
}
# Transposed-operand variants: name -> (workload, A stored K x M, B stored N x K).
# The same seeded matrices, stored transposed in HBM.
TRANSPOSED = {
    "bf16_gemm_8192_ta": ("bf16_gemm_8192", True, False),
    "bf16_gemm_8192_tb": ("bf16_gemm_8192", False, True),
    "bf16_gemm_8192_tatb": ("bf16_gemm_8192", True, True),
    "bf16_gemm_16x8192x8192_tb": ("bf16_gemm_16x8192x8192", False, True),
    "bf16_gemm_128x14336x4096_tb": ("bf16_gemm_128x14336x4096", False, True),
}
HEADLINE = "bf16_gemm_8192"
BREAKDOWN = [w for w in WORKLOADS if w != HEADLINE] + list(TRANSPOSED)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def ffma_peak_tflops(mhz):
    """fp32 FMA peak: SMs x 128 lanes x 2 flops x clock (MHz)."""
    return N_SMS_B200 * FFMA_LANES_PER_SM * 2 * mhz * 1e6 / 1e12


def make_inputs(name):
    """Seeded host inputs (numpy stored values) of a workload."""
    kind, M, N, K, seed, relu, dist = WORKLOADS[name]
    if kind == "w4a16":
        A, Bq, S, _ = synth.w4a16(M, N, K, seed)
        return {"A": A, "Bq": Bq, "S": S}
    if kind == "wfp4":
        A, Bq, E, _ = synth.wfp4(M, N, K, seed)
        return {"A": A, "Bq": Bq, "S": E}
    if kind == "sp24_bf16":
        Ac, E, B, _ = synth.sp24(M, N, K, seed, "bf16")
        return {"A": Ac, "E": E, "B": B}
    st = {"bf16": "bf16", "f16": "f16"}.get(kind, "f32")
    if dist == "normal_sqrtk":
        A, B = synth.normal(M, N, K, seed, st, scale_by_sqrt_k=True)
    else:
        A, B = synth.normal(M, N, K, seed, st)
    return {"A": A, "B": B}


def _torch_of(arr, kind, device, pinned=False):
    """numpy stored values -> torch tensor with a 16-byte-multiple row pitch."""
    import torch
    rows, cols = arr.shape
    eb = arr.dtype.itemsize
    per = 16 // eb
    ld = max(per, -(-cols // per) * per)
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16,
           "u8": torch.uint8}[kind]
    host = np.zeros((rows, ld), arr.dtype)
    host[:, :cols] = arr
    if arr.dtype == np.uint16:
        t = torch.from_numpy(host.view(np.int16)).view(tdt)
    else:
        t = torch.from_numpy(host)
    if device == "cpu":
        t = t.pin_memory() if pinned else t
    else:
        t = t.to(device)
    return t[:, :cols]


def _empty_out(M, N, tdt, device, pinned=False):
    import torch
    eb = torch.tensor([], dtype=tdt).element_size()
    per = 16 // eb
    ld = max(per, -(-N // per) * per)
    t = torch.empty((M, ld), dtype=tdt, device=device, pin_memory=pinned and device == "cpu")
    return t[:, :N]


def workload_facts(name, peaks):
    """Algorithmic work of one launch of a workload and the roofline that
    bounds it: (flops, alg_bytes, bound, peak, unit).

    flops = 2*M*N*K.  alg_bytes = each operand read once plus C written once:
    2 or 4 bytes per element, and for the 4-bit paths the packed weights
    (ceil(N/2) bytes per row of K) and the scales: (K/128) x N fp16, or
    ceil(K/32) x N E8M0 bytes for FP4 weights.  Padded
    MMA work and dequantisation arithmetic are not counted.  A contraction
    whose flops per byte lie below the ridge (tensor peak / HBM bandwidth)
    is HBM-bound; the fp32 FFMA path is bound by the FMA pipe ("alu"); TF32
    takes the bf16 peak times the nominal dense ratio 1.1 / 2.25.  The 2:4
    sparse GEMM counts the multiply-adds its kept values need (M*N*K flops,
    half the dense count) and the compressed A (K/2 values and K/8 code
    bytes per row), against the dense bf16 peak: the sparse tensor cores do
    the same multiply-adds per cycle on half the operands."""
    base = TRANSPOSED.get(name, (name, False, False))[0]
    kind, M, N, K = WORKLOADS[base][:4]
    flops = 2.0 * M * N * K
    if kind == "sp24_bf16":
        flops = float(M) * N * K
        alg_bytes = M * (K // 2) * 2 + M * ((K + 7) // 8) + K * N * 2 + M * N * 2
    elif kind == "w4a16":
        alg_bytes = M * K * 2 + K * ((N + 1) // 2) + (K // 128) * N * 2 + M * N * 2
    elif kind == "wfp4":
        alg_bytes = M * K * 2 + K * ((N + 1) // 2) + ((K + 31) // 32) * N + M * N * 2
    else:
        eb = 2 if kind in ("bf16", "f16") else 4
        alg_bytes = (M * K + K * N + M * N) * eb
    tensor_peak = peaks["bf16_tflops"]
    if kind == "f32_tf32":
        tensor_peak *= 1.1 / 2.25
    ridge = tensor_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if kind == "f32_ffma":
        return flops, alg_bytes, "alu", ffma_peak_tflops(peaks.get("sm_max_mhz", 1965.0)), "TFLOP/s"
    if flops / alg_bytes < ridge:
        return flops, alg_bytes, "hbm", peaks["hbm_gbs"], "GB/s"
    return flops, alg_bytes, "tensor", tensor_peak, "TFLOP/s"


class Case:
    """A workload bound to device buffers, with its roofline facts."""

    def __init__(self, name, device, peaks):
        import torch
        import tiled_dense_gemm_tma_b200 as tg
        self.name = name
        base, ta, tb = TRANSPOSED.get(name, (name, False, False))
        kind, M, N, K, seed, relu, dist = WORKLOADS[base]
        self.kind, self.M, self.N, self.K, self.relu = kind, M, N, K, relu
        self.trans = (ta, tb)
        host = make_inputs(base)
        if ta:
            host["A"] = np.ascontiguousarray(host["A"].T)
        if tb:
            host["B"] = np.ascontiguousarray(host["B"].T)
        self.flops, self.alg_bytes, self.bound, self.peak, self.unit = workload_facts(name, peaks)
        if kind == "w4a16":
            self.A = _torch_of(host["A"], "f16", device)
            self.Bq = _torch_of(host["Bq"], "u8", device)
            self.S = _torch_of(host["S"], "f16", device)
            self.C = _empty_out(M, N, torch.float16, device)
            self.dtype = "f16 x int4"
            self._host = host
            self.run = lambda: tg.gemm_w4a16(self.A, self.Bq, self.S, N, C=self.C, relu=relu)
        elif kind == "sp24_bf16":
            self.A = _torch_of(host["A"], "bf16", device)
            self.E = _torch_of(host["E"], "u8", device)
            self.B = _torch_of(host["B"], "bf16", device)
            self.C = _empty_out(M, N, torch.bfloat16, device)
            self.dtype = "bf16 (A 2:4 sparse)"
            self._host = host
            self.run = lambda: tg.gemm_sp24(self.A, self.E, self.B, C=self.C, relu=relu)
        elif kind == "wfp4":
            self.A = _torch_of(host["A"], "bf16", device)
            self.Bq = _torch_of(host["Bq"], "u8", device)
            self.S = _torch_of(host["S"], "u8", device)
            self.C = _empty_out(M, N, torch.bfloat16, device)
            self.dtype = "bf16 x fp4 (e2m1, e8m0 per 32 k)"
            self._host = host
            self.run = lambda: tg.gemm_wfp4(self.A, self.Bq, self.S, N, C=self.C, relu=relu)
        else:
            ik = {"bf16": "bf16", "f16": "f16"}.get(kind, "f32")
            tdt = {"bf16": torch.bfloat16, "f16": torch.float16}.get(kind, torch.float32)
            self.A = _torch_of(host["A"], ik, device)
            self.B = _torch_of(host["B"], ik, device)
            self.C = _empty_out(M, N, tdt, device)
            self.dtype = {"bf16": "bf16", "f16": "f16", "f32_ffma": "f32", "f32_tf32": "tf32"}[kind]
            self._host = host
            self._ik = ik
            if kind == "bf16":
                self.run = lambda: tg.gemm_bf16(self.A, self.B, C=self.C, relu=relu,
                                                trans_a=ta, trans_b=tb)
            elif kind == "f16":
                self.run = lambda: tg.gemm_f16(self.A, self.B, C=self.C, relu=relu,
                                               trans_a=ta, trans_b=tb)
            else:
                mode = tg.F32_TF32 if kind == "f32_tf32" else tg.F32_FFMA
                self.run = lambda: tg.gemm_f32(self.A, self.B, C=self.C, relu=relu, mode=mode)

    def achieved(self, seconds):
        if self.unit == "GB/s":
            return self.alg_bytes / seconds / 1e9
        return self.flops / seconds / 1e12

    def host_pinned(self):
        """Pinned host copies of the inputs, by the name of the device input
        they feed, and a pinned host output (e2e)."""
        if self.kind == "sp24_bf16":
            pairs = [("A", _torch_of(self._host["A"], "bf16", "cpu", pinned=True)),
                     ("E", _torch_of(self._host["E"], "u8", "cpu", pinned=True)),
                     ("B", _torch_of(self._host["B"], "bf16", "cpu", pinned=True))]
            return pairs, _empty_out(self.M, self.N, self.C.dtype, "cpu", pinned=True)
        if self.kind in ("w4a16", "wfp4"):
            ak, sk = ("f16", "f16") if self.kind == "w4a16" else ("bf16", "u8")
            hA = _torch_of(self._host["A"], ak, "cpu", pinned=True)
            hB = _torch_of(self._host["Bq"], "u8", "cpu", pinned=True)
            hS = _torch_of(self._host["S"], sk, "cpu", pinned=True)
            return [("A", hA), ("Bq", hB), ("S", hS)], \
                _empty_out(self.M, self.N, self.C.dtype, "cpu", pinned=True)
        hA = _torch_of(self._host["A"], self._ik, "cpu", pinned=True)
        hB = _torch_of(self._host["B"], self._ik, "cpu", pinned=True)
        return [("A", hA), ("B", hB)], _empty_out(self.M, self.N, self.C.dtype, "cpu",
                                                  pinned=True)


# ------------------------------------------------------------------ timing

class ClockSampler:
    """Samples the GPU's SM clock, power and clock-event reasons while the
    timed region runs.  Read-only NVML queries from a background thread every
    millisecond, each sample stamped with the host clock; the GPU is found by
    the CUDA device's PCI address, so the sampled GPU is the one the bench
    runs on whatever the visible-device mapping.  summary() reports the
    samples taken between the host times that bracket the timed region (the
    GPU runs the region's launches between them).  Falls back to
    `nvidia-smi -lms 100` when NVML is unavailable."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.001

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.thread = None
        self.rows = []
        self.stop = False

    def _bus_id(self):
        import torch
        prop = torch.cuda.get_device_properties(self.gpu)
        return f"{prop.pci_domain_id:08X}:{prop.pci_bus_id:02X}:{prop.pci_device_id:02X}.0"

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(self._bus_id())

    def _poll(self, nv, h):
        bits = [nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap]
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.rows.append(["0", str(sm), str(mx), str(pw), hex(r)] +
                                 ["Active" if r & b else "Not Active" for b in bits] +
                                 [time.time()])
            except Exception:                        # stop sampling, keep what we have
                return
            time.sleep(self.PERIOD_S)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.thread.start()
            t0 = time.time()
            while not self.rows and time.time() - t0 < 2.0:
                time.sleep(0.005)
            return self
        except Exception:
            self.thread = None
        import tempfile
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self._bus_id(), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            t0 = time.time()                 # wait for the first sample
            while os.path.getsize(self.path) == 0 and time.time() - t0 < 5.0:
                time.sleep(0.05)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop = True
            self.thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, window=None):
        """Clock record; with window = (t0, t1) host times, only the samples
        taken inside it (all samples when none fell inside)."""
        rows = list(self.rows)
        in_window = None
        if window is not None:
            t0, t1 = window
            inside = [r for r in rows if len(r) > 9 and t0 <= r[9] <= t1]
            in_window = len(inside)
            if inside:
                rows = inside
        if self.path and os.path.exists(self.path):
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.remove(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].lower().startswith("active")})
        # samples under load: power well above idle
        loaded = [s for s, p in zip(sm, pw) if p is not None and pw and p > 0.5 * max(pw)] or sm
        return {"sm_mhz": float(np.median(loaded)) if loaded else None,
                "sm_mhz_mean": round(float(np.mean(loaded)), 1) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "samples": len(rows), "samples_in_timed_region": in_window,
                "period_ms": self.PERIOD_S * 1e3, "reasons": reasons}


def flush_l2(bufs):
    """Evict L2: write a buffer larger than L2, then read a second one, so the
    lines left in L2 are clean and the timed launch pays no write-backs."""
    wbuf, rbuf, sink = bufs
    wbuf.add_(1)
    torch_sum = rbuf.sum(dtype=None)
    sink.copy_(torch_sum)


def time_breakdown(case, iters, warmup, flush_buf):
    """Per-launch device time (s), flushing L2 before each launch: (median,
    min, trimmed mean).  A launch's two event stamps land on a coarse grid on
    these devices (steps of about 2 us at the end of short kernels), so the
    median of a short kernel snaps to that grid; the mean over the launches,
    whose phase against the grid varies, does not.  The mean is taken over
    the middle 80 % of the sorted times, so a rare slow launch (a clock dip,
    another process) does not move it; it is the estimate the rates use."""
    import torch
    for _ in range(warmup):
        case.run()
    torch.cuda.synchronize()
    ts = []
    for _ in range(iters):
        flush_l2(flush_buf)
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record()
        case.run()
        e.record()
        e.synchronize()
        ts.append(s.elapsed_time(e) * 1e-3)
    srt = np.sort(np.asarray(ts))
    cut = len(srt) // 10
    mid = srt[cut:len(srt) - cut] if len(srt) > 2 * cut else srt
    return float(np.median(srt)), float(srt[0]), float(np.mean(mid))


def traffic_record(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if the kernel
    sources are unchanged since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    src = source_digest()
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if len(line) == 3 and line[0] == kernel_key and line[1] == src:
                return float(line[2])
    return None


# Sources the headline (tensor-core, 16-bit) kernel is built from; its DRAM
# traffic figure stays valid while these are unchanged.
HEADLINE_SOURCES = ("ptx.cuh", "tile_sched.h", "host.cuh", "host.cu", "launch.h", "gemm_tc.cuh", "gemm_tc2.cuh",
                    "gemm_tc.cu")


def source_digest(files=HEADLINE_SOURCES):
    """Short digest of the given CUDA sources (identifies the kernel build)."""
    h = hashlib.sha256()
    for name in sorted(files):
        with open(os.path.join(ROOT, "tiled_dense_gemm_tma_b200", "csrc", name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:12]


# ------------------------------------------------------------ CPU oracle leg

def oracle_block(name, host, rows, cols):
    """Run the fp64 oracle on the block C[rows, cols] (full K); return seconds."""
    import oracle
    kind = WORKLOADS[name][0]
    if kind in ("w4a16", "wfp4"):
        A = np.ascontiguousarray(host["A"][rows])
        ncols = len(cols)
        c0 = int(cols[0]) & ~1
        Bq = np.ascontiguousarray(host["Bq"][:, c0 // 2:(c0 + ncols + 1) // 2 + 1])
        S = np.ascontiguousarray(host["S"][:, c0:c0 + ncols])
        fn = oracle.gemm_w4a16 if kind == "w4a16" else oracle.gemm_wfp4
        t0 = time.perf_counter()
        fn(A, Bq, S, N=ncols)
        return time.perf_counter() - t0
    if kind == "sp24_bf16":
        Ac = np.ascontiguousarray(host["A"][rows])
        E = np.ascontiguousarray(host["E"][rows])
        B = np.ascontiguousarray(host["B"][:, cols])
        t0 = time.perf_counter()
        oracle.gemm_sp24(Ac, E, B, "bf16")
        return time.perf_counter() - t0
    A = np.ascontiguousarray(host["A"][rows])
    B = np.ascontiguousarray(host["B"][:, cols])
    fn = {"bf16": oracle.gemm_bf16, "f16": oracle.gemm_f16}.get(kind, oracle.gemm_f32)
    t0 = time.perf_counter()
    fn(A, B)
    return time.perf_counter() - t0


def oracle_rate(name, host, budget_s):
    """Calibrate, then time the oracle on a block sized to ~budget_s seconds.
    Returns (flops/s, description of the sample, threads)."""
    import oracle
    kind, M, N, K = WORKLOADS[name][:4]
    cols = np.arange(min(N, 256))
    r = max(1, min(M, 2 * oracle.num_threads()))
    t = oracle_block(name, host, np.arange(r), cols)
    per_out = t / (r * len(cols))
    r2 = int(max(1, min(M, budget_s / per_out / len(cols))))
    rows = np.arange(r2)
    t = oracle_block(name, host, rows, cols)
    flops = 2.0 * r2 * len(cols) * K
    desc = f"C[0:{r2}, 0:{len(cols)}] of the {M}x{N}x{K} workload (full K), one oracle call"
    return flops / t, desc, oracle.num_threads(), t


# ------------------------------------------------------------ offline sweep
#
# Shape classes of the tuning table: (op, m_lo, m_hi, n_lo, n_hi), the
# configured workloads that represent the class, and the candidate launch
# shapes timed for it.  The all-default candidate is always timed first; a
# class gets a built-in rule only when another candidate beats it by more
# than SWEEP_MARGIN on the geometric mean of its workloads' times.
INF = (1 << 63) - 1
_PAIR16 = ([{"path": "cta_pair", "stages": st, "group_m": g} for st in (4, 6) for g in (4, 8, 16)] +
           [{"path": "one_cta", "group_m": g} for g in (8, 16)])
_SMALL = [{"path": "small_m", "ctas": c} for c in (140, 128, 120, 112, 104, 96, 74)]
# (the small-M classes are measured on wide weight matrices only, so their
# rules cover N >= 4096; narrower N keeps the defaults)
SWEEP_CLASSES = [
    ("bf16", 5, 64, 4096, INF, ["bf16_gemm_16x8192x8192"], _SMALL + [{"path": "cta_pair"}]),
    ("bf16", 65, 128, 4096, INF, ["bf16_gemm_128x14336x4096"], _SMALL + [{"path": "cta_pair"}]),
    ("bf16", 129, INF, 1, INF, ["bf16_gemm_8192", "bf16_gemm_4096", "bf16_gemm_8192x1024x8192",
                                "bf16_gemm_3000x5000x4000"], _PAIR16),
    ("f16", 129, INF, 1, INF, ["f16_gemm_8192", "f16_gemm_4096_relu"], _PAIR16),
    ("w4a16", 1, 4, 4096, INF, ["w4a16_gemm_m1"],
     [{"path": "cuda_core", "ctas": c} for c in (136, 128, 120, 96)] + [{"path": "small_m"}] +
     _SMALL[2:]),
    ("w4a16", 5, 128, 4096, INF, ["w4a16_gemm_m16"], _SMALL),
    ("w4a16", 129, INF, 1, INF, ["w4a16_gemm_m4096"],
     [{"path": "cta_pair", "group_m": g} for g in (4, 16)] + [{"path": "one_cta"}]),
    ("wfp4", 1, 4, 4096, INF, ["wfp4_gemm_m1"],
     [{"path": "cuda_core", "ctas": c} for c in (136, 128, 120, 96)] + [{"path": "small_m"}]),
    ("wfp4", 5, 128, 4096, INF, ["wfp4_gemm_m16"], _SMALL),
    ("wfp4", 129, INF, 1, INF, ["wfp4_gemm_m4096"],
     [{"path": "cta_pair", "group_m": g} for g in (4, 16)] + [{"path": "one_cta"}]),
    ("f32_ffma", 1, 1024, 1, 1024, ["f32_ffma_gemm_1024"], [{"splits": k} for k in (1, 3, 4)]),
    ("f32_tf32", 129, INF, 1, INF, ["f32_tf32_gemm_4096"],
     [{"group_m": g} for g in (4, 16)] + [{"path": "one_cta"}]),
]
SWEEP_MARGIN = 0.02
TUNE_TABLE = os.path.join(ROOT, "tiled_dense_gemm_tma_b200", "csrc", "tune_table.h")
SWEEP_REPORT = os.path.join(ROOT, "profiles", "tune_sweep.md")
_RULE_FIELDS = ("op", "path", "m_lo", "m_hi", "n_lo", "n_hi", "ctas", "group_m", "splits",
                "stages")


def sweep_pick(times, margin=SWEEP_MARGIN):
    """times: one list of per-workload seconds per candidate (candidate 0 is
    the default).  Returns the index of the candidate with the smallest
    geometric mean, or 0 unless it beats the default by more than margin."""
    gm = [float(np.exp(np.mean(np.log(t)))) for t in times]
    best = int(np.argmin(gm))
    return best if gm[best] < gm[0] * (1.0 - margin) else 0


def tune_table_source(rules, notes):
    """C++ source of tune_table.h for the chosen rules (dicts of numbers)."""
    lines = ["// tune_table.h -- built-in tuning rules (see tune.h).  Written by",
             "// `python bench.py --sweep` on one B200 from the timings in",
             "// profiles/tune_sweep.md; a class without a rule keeps every default.",
             "#pragma once", '#include "tune.h"', "", "namespace tg {", "",
             "constexpr TuneRule kBuiltinRules[] = {"]
    for r, note in zip(rules, notes):
        vals = ", ".join(("0x7fffffffffffffffll" if r[f] == INF else str(int(r[f])))
                         for f in _RULE_FIELDS)
        lines.append(f"    {{{vals}}},   // {note}")
    lines += ["    {-1, 0, 0, 0, 0, 0, 0, 0, 0, 0},   // end: matches nothing", "};", "",
              "}  // namespace tg", ""]
    return "\n".join(lines)


def run_sweep(args):
    """Time every candidate of every class on this GPU; write the built-in
    rules (tune_table.h) and the report (profiles/tune_sweep.md)."""
    import torch
    import tiled_dense_gemm_tma_b200 as tg
    dev = torch.device("cuda", 0)
    tg.load_library()
    peaks, _ = load_peaks()
    flush = (torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev),
             torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev),
             torch.zeros((), dtype=torch.float32, device=dev))
    chosen, notes = [], []
    report = ["# Offline tile / stage sweep (tuning table)", "",
              "Command: `python bench.py --sweep` on one B200.  Each candidate is timed",
              f"as the trimmed mean (middle 80 %) of {args.breakdown_iters} launches per workload, L2 flushed "
              "before each launch; the default is the library's choice with no rule.  A class",
              f"takes a rule when its best candidate's geometric-mean time is more than "
              f"{SWEEP_MARGIN:.0%} below the default's.", ""]
    tg.tune_set([])
    for op, m_lo, m_hi, n_lo, n_hi, wls, cands in SWEEP_CLASSES:
        cases = [Case(w, dev, peaks) for w in wls]
        base = {"op": op, "m_lo": m_lo, "m_hi": m_hi, "n_lo": n_lo, "n_hi": n_hi}
        allc = [{}] + list(cands)
        times = []
        for cand in allc:
            # the default too runs under a rule of the class, with every field
            # at its default: it masks the built-in rules, which a sweep must
            # not take as the default it measures against
            tg.tune_set([dict(base, **cand)])
            row = []
            for c in cases:
                _, _, med = time_breakdown(c, args.breakdown_iters, 10, flush)
                if tg.last_device_status() != 0:
                    raise RuntimeError(f"device status after {op} {cand}")
                row.append(med)
            times.append(row)
        tg.tune_set([])
        best = sweep_pick(times)
        cls = f"{op} M {m_lo}..{'inf' if m_hi == INF else m_hi}"
        report += [f"## {cls}", "", "| candidate | " + " | ".join(f"{w} (us)" for w in wls) +
                   " | geo-mean vs default |", "|---|" + "---|" * (len(wls) + 1)]
        gm0 = float(np.exp(np.mean(np.log(times[0]))))
        for i, (cand, row) in enumerate(zip(allc, times)):
            gm = float(np.exp(np.mean(np.log(row))))
            name = ", ".join(f"{k}={v}" for k, v in cand.items()) or "default"
            mark = " **chosen**" if i == best else ""
            report.append(f"| {name}{mark} | " + " | ".join(f"{t * 1e6:.2f}" for t in row) +
                          f" | {gm / gm0:.3f} |")
        report.append("")
        if best:
            r = {f: 0 for f in _RULE_FIELDS}
            r.update(base)
            r.update(allc[best])
            r["op"] = tg.OPS[op]
            r["path"] = tg.PATHS[r["path"]] if isinstance(r["path"], str) else r["path"]
            chosen.append(r)
            notes.append(f"{cls}: " + ", ".join(f"{k}={v}" for k, v in allc[best].items()) +
                         f" ({float(np.exp(np.mean(np.log(times[best])))) / gm0:.3f} of the default)")
        del cases
        torch.cuda.empty_cache()
    with open(TUNE_TABLE, "w") as f:
        f.write(tune_table_source(chosen, notes))
    with open(SWEEP_REPORT, "w") as f:
        f.write("\n".join(report) + "\n")
    print(json.dumps({"sweep": "done", "rules": len(chosen), "table": TUNE_TABLE,
                      "report": SWEEP_REPORT}), flush=True)
    return 0


# ------------------------------------------------------------------- main

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-breakdown", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--breakdown-iters", type=int, default=50)
    ap.add_argument("--sweep", action="store_true",
                    help="time the tuning table's candidates and rewrite its built-in rules")
    return ap.parse_args()


def max_over_ranks(group, x, device):
    """Largest value of x over all ranks (x itself when there is one rank)."""
    if group is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    group.all_reduce(t, op=group.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank_step, steps, world, elapsed_max_s):
    """Whole-job throughput: every rank processes the same units per step
    (independent problems, weak scaling); the job takes as long as its
    slowest rank."""
    return units_per_rank_step * steps * world / elapsed_max_s


def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


METRIC = "GEMM TFLOP/s and % of sm_100a dense peak per dtype at 4096\u00b3/8192\u00b3, 1\u00d7B200"


def metric_name():
    """The headline metric's name (TFLOP/s, and the fraction of the sm_100a
    dense peak for the dtype)."""
    return METRIC


def run_reference(args, ws, rank):
    """CPU oracle timed as the reference arm (rank 0 only)."""
    if rank != 0:
        return 0
    name = args.workload
    host = make_inputs(name)
    total_budget = 150.0
    per_step = max(0.05, total_budget / max(1, args.steps + args.warmup))
    import oracle
    kind, M, N, K = WORKLOADS[name][:4]
    cols = np.arange(min(N, 256))
    r0 = max(1, min(M, 2 * oracle.num_threads()))
    t = oracle_block(name, host, np.arange(r0), cols)      # calibration
    per_step = min(per_step, 30.0)
    r = int(max(1, min(M, per_step / (t / (r0 * len(cols))) / len(cols))))
    for _ in range(args.warmup):
        oracle_block(name, host, np.arange(r), cols)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_block(name, host, np.arange(r), cols)
    el = time.perf_counter() - t0
    flops = 2.0 * r * len(cols) * K * args.steps
    value = flops / el / 1e12
    sample = f"each step: C[0:{r}, 0:{len(cols)}] of the {M}x{N}x{K} workload (full K)"
    line = {"impl": "reference", "metric": metric_name(), "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": name, "M": M, "N": N, "K": K},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    ws, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_reference(args, ws, rank)
    if args.sweep:
        return run_sweep(args)

    import torch
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    group = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        group = dist
    import tiled_dense_gemm_tma_b200 as tg
    tg.load_library()
    peaks, peak_src = load_peaks()

    def barrier():
        if group is not None:
            group.barrier()


    # ---------------------------------------------------------- headline
    case = Case(args.workload, dev, peaks)
    case.run()
    torch.cuda.synchronize()
    st = tg.last_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after first launch")
    for _ in range(args.warmup):
        case.run()
    K = args.steps
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        h0 = time.time()
        t_start.record()
        for i in range(K):
            ev_s[i].record()
            case.run()
            ev_e[i].record()
        t_end.record()
        torch.cuda.synchronize()
        h1 = time.time()
        barrier()
    clocks = clk.summary(window=(h0, h1))
    elapsed = max_over_ranks(group, t_start.elapsed_time(t_end) * 1e-3, dev)
    launch_s = float(np.mean([a.elapsed_time(b) for a, b in zip(ev_s, ev_e)])) * 1e-3
    st = tg.last_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} in timed region")
    value = job_rate(case.flops, K, ws, elapsed) / 1e12      # whole-job TFLOP/s

    # -------------------------------------------------------------- e2e
    # Each step uploads its inputs from pinned host memory, runs the GEMM
    # through the public binding and downloads C, all inside the timed
    # region.  Consecutive steps are pipelined over three streams and two
    # device copies of the operands: step i+1's upload and step i-1's
    # download run while step i computes.
    pairs, host_out = case.host_pinned()
    n_e2e = max(3, min(K, 20))
    h2d = sum(h._base.numel() * h._base.element_size() for _, h in pairs)
    d2h = host_out._base.numel() * host_out._base.element_size()
    names = [n for n, _ in pairs] + ["C"]

    def twin(t):
        return torch.empty_like(t._base)[:, :t.shape[1]]
    sets = [{n: getattr(case, n) for n in names}, {n: twin(getattr(case, n)) for n in names}]
    s_comp = torch.cuda.current_stream()
    s_up, s_dn = torch.cuda.Stream(), torch.cuda.Stream()
    up_done = [torch.cuda.Event(), torch.cuda.Event()]
    comp_done = [torch.cuda.Event(), torch.cuda.Event()]
    dn_done = [torch.cuda.Event(), torch.cuda.Event()]

    def e2e_step(i):
        st = sets[i % 2]
        s_up.wait_event(comp_done[i % 2])         # the GEMM two steps back has read this set
        with torch.cuda.stream(s_up):
            for n, h in pairs:
                st[n]._base.copy_(h._base, non_blocking=True)
            up_done[i % 2].record(s_up)
        s_comp.wait_event(up_done[i % 2])
        s_comp.wait_event(dn_done[i % 2])         # this set's previous C has been read back
        for n in names:
            setattr(case, n, st[n])
        case.run()
        comp_done[i % 2].record(s_comp)
        s_dn.wait_event(comp_done[i % 2])
        with torch.cuda.stream(s_dn):
            host_out._base.copy_(st["C"]._base, non_blocking=True)
            dn_done[i % 2].record(s_dn)
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_comp)
    s_up.wait_event(e0)
    s_dn.wait_event(e0)
    for i in range(n_e2e):
        e2e_step(i)
    s_comp.wait_event(dn_done[(n_e2e - 1) % 2])
    e1.record(s_comp)
    torch.cuda.synchronize()
    barrier()
    for n in names:
        setattr(case, n, sets[0][n])
    e2e_s = max_over_ranks(group, e0.elapsed_time(e1) * 1e-3, dev)
    e2e_val = job_rate(case.flops, n_e2e, ws, e2e_s) / 1e12

    # -------------------------------------------------------- breakdown
    breakdown = []
    if not args.no_breakdown and ws == 1:
        flush = (torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev),
                 torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev),
                 torch.zeros((), dtype=torch.float32, device=dev))
        del case.A
        for name in BREAKDOWN:
            try:
                c = Case(name, dev, peaks)
                c.run()
                torch.cuda.synchronize()
                med, mn, mean = time_breakdown(c, args.breakdown_iters, 10, flush)
                ok = tg.last_device_status() == 0
                breakdown.append({"workload": name, "dtype": c.dtype,
                                  "tflops": round(c.flops / mean / 1e12, 2),
                                  "gbs": round(c.alg_bytes / mean / 1e9, 1),
                                  "us_mean": round(mean * 1e6, 2),   # middle 80 % of the launches
                                  "us_median": round(med * 1e6, 2), "us_min": round(mn * 1e6, 2),
                                  "bound": c.bound, "frac": round(c.achieved(mean) / c.peak, 4),
                                  "peak": round(c.peak, 1), "peak_unit": c.unit,
                                  "status_ok": ok, "l2": "flushed (write + clean read of 512 MB) before each launch"})
                del c
            except Exception as exc:           # report, never hide
                breakdown.append({"workload": name, "error": str(exc)[:200]})
            torch.cuda.empty_cache()
        del flush

    # ------------------------------------------------------ cpu baseline
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rate, desc, threads, t = oracle_rate(args.workload, case._host, 15.0)
        cpu = {"value": rate / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": desc + f" ({t:.1f} s)"}

    if rank == 0:
        kind, M, N, Kd, seed, relu, dist_name = WORKLOADS[args.workload]
        traffic = traffic_record(args.workload)
        achieved = case.achieved(launch_s)
        # the same peak measured as a seconds-long loop under the power cap
        sustained = None
        if case.unit == "TFLOP/s" and case.bound == "tensor" and "bf16_tflops_sustained" in peaks:
            sustained = round(case.peak * peaks["bf16_tflops_sustained"] / peaks["bf16_tflops"], 1)
        line = {
            "metric": metric_name(), "value": round(value, 3), "unit": "TFLOP/s",
            "n_gpus": ws, "steps": K, "warmup": args.warmup,
            "ms_per_step": round(elapsed / K * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": case.dtype,
            "data": "synthetic (seeded; N(0,1)/sqrt(K) entries)",
            "config": {"workload": args.workload, "M": M, "N": N, "K": Kd, "seed": seed,
                       "relu": relu, "parallelism": f"independent GEMM per GPU x{ws}",
                       "l2": "inputs (256 MB) larger than L2; back-to-back launches"},
            "roofline": {"bound": case.bound, "achieved": round(achieved, 2),
                         "peak": case.peak, "unit": case.unit,
                         "frac": round(achieved / case.peak, 4),
                         "sm_mhz_mean": clocks.get("sm_mhz_mean"),
                         "traffic": traffic, "peak_source": f"{peak_src} (burst)",
                         "peak_sustained": sustained,
                         "frac_of_sustained": (round(achieved / sustained, 4) if sustained else None),
                         "algorithmic_per_launch": case.flops if case.unit == "TFLOP/s"
                         else case.alg_bytes},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_val, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": n_e2e,
                    "overlap": "upload of step i+1 and download of step i-1 beside the GEMM of "
                               "step i (three streams, two device copies of the operands)"},
            "gpu_launches": K,
            "clocks": clocks,
            "kernel_source": source_digest(),
            "breakdown": breakdown,
        }
        print(json.dumps(line), flush=True)
    if group is not None:
        group.barrier()
        group.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
