"""Benchmark of the W4A4 NVFP4 hot path on B200.

One step = one pass of the per-call hot path over one batch of synthetic
prefill activations:  fp4_quantize_act (amax pass + fused block quantizer,
DYNAMIC global scale, MMA scale order)  ->  fp4_gemm (tcgen05 block-scaled
GEMM, alpha epilogue, bf16 out).  Weights are quantized once before timing
(fp4_quantize_weights, the load-time step).

Workload: M=8192, N=28672, K=8192 (the large prefill GEMM), A ~ N(0,1) with
0.1% of entries x100, W ~ N(0,0.02).  Inputs exceed L2 (A 128 MiB, packed W
131 MiB, C 448 MiB), so no explicit flush is needed between steps.

Beside the headline step the JSON line carries: the prefill matrix (M in
{2048, 8192} x (N, K) in {(8192, 8192), (28672, 8192)}, NVFP4 bf16 / fp32
out and MXFP4, GEMM alone and quantize + GEMM), the decode shapes through
the fused entry point, the activation-quantize sweep, the synthetic 24-layer
decoder against bf16, the vendor FP4 GEMM on the same operands (context),
and the CPU oracle's three baseline legs (prefill GEMM row sample, quantize
sweep on all cores and one core, decode shapes in full).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun each rank runs an independent replica on its own GPU (the
path has no exchange step); the value is total FLOPs over the max per-rank
time.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DECODE_SHAPES = [(M, N, K) for (N, K) in ((4096, 4096), (14336, 4096), (4096, 14336))
                 for M in (1, 8, 32)]
SWEEP_SHAPES = [(M, K) for M in (1, 32, 512, 8192) for K in (2880, 8192, 16384)]
L2_BYTES = 126 * 2 ** 20

M, N, K = 8192, 28672, 8192
FLOP = 2.0 * M * N * K
METRIC = "NVFP4 GEMM TFLOPS (% of B200 FP4 peak); quantize GB/s (% of HBM)"
WORKLOAD = "prefill W4A4 NVFP4 GEMM M=8192 N=28672 K=8192, bf16 out, activation quantized per step"
# algorithmic bytes per activation element of the DYNAMIC quantizer:
# amax pass reads 2 B; quantize pass reads 2 B, writes 0.5 B codes + 1/16 B scales
QUANT_BYTES_PER_ELEM = 2.0 + 2.0 + 0.5 + 1.0 / 16.0
FP4_OVER_BF16 = 4.0     # nominal dense FP4 / dense BF16 tensor throughput on B200 (9 / 2.25)
FP4_NOMINAL_TFLOPS = 9000.0   # B200 dense FP4 tensor peak, nominal (context)
# DRAM read + write bytes of one launch of the GEMM kernel the bench shape
# takes (gemm_pair_kernel), measured with ncu (dram__bytes_read.sum +
# dram__bytes_write.sum, one pass).  None whenever that kernel has changed
# since it was last measured.
GEMM_TRAFFIC_BYTES = 264.9e6 + 441.7e6


def gemm_kernel_name(m, n, k):
    """The GEMM kernel fp4_gemm launches for this shape (fp4_gemm_plan)."""
    from mxfp4_block_scaled_fp4_b200 import ops
    tm, tn, sp = ops.gemm_plan(m, n, k, 0)
    if tm == 256:
        return "fp4 gemm_pair_kernel (tcgen05 cta_group::2 kind::mxf4nvf4, 256x256 tiles)"
    return (f"fp4 gemm_kernel (tcgen05 cta_group::1 kind::mxf4nvf4, {tm}x{tn} tiles"
            + (f", K split over {sp}-CTA clusters)" if sp > 1 else ")"))


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class Clocks:
    """SM clocks and throttle reasons sampled DURING a region: an NVML thread
    (reads only) every ~1 ms, so that even a region of a few milliseconds
    gets samples; nvidia-smi's 200 ms loop runs beside it as a second
    record.  Nothing is set on the GPU."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80),
               ("sw_power_cap", 0x4))

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None
        self.thread = None
        self.samples = []
        self.stop_flag = False
        self.nvml_err = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            pr = torch.cuda.get_device_properties(self.dev)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def _loop(self, h):
        import pynvml
        smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stop_flag:
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.perf_counter(), sm, smax, rs))
            except Exception as e:  # keep the region's timing intact
                self.nvml_err = str(e)[:80]
                return
            time.sleep(0.001)

    def start(self):
        """Starts the samplers and returns once the NVML thread is taking
        samples (its first calls can take longer than a short region)."""
        import threading
        try:
            h = self._handle()
            self.thread = threading.Thread(target=self._loop, args=(h,), daemon=True)
            self.thread.start()
            t_end = time.perf_counter() + 2.0
            while not self.samples and self.nvml_err is None and time.perf_counter() < t_end:
                time.sleep(0.001)
        except Exception as e:
            self.nvml_err = f"{type(e).__name__}: {str(e)[:80]}"
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        self.t0 = time.perf_counter()

    def _smi(self):
        if self.proc is None:
            return []
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]),
                                 {nm for nm, v in zip(names, parts[5:9]) if v.lower() == "active"}))
                except ValueError:
                    continue
        os.unlink(self.path)
        return rows

    def stop(self):
        """Summary of the samples taken between start() and stop(); a region
        shorter than one NVML round trip gets the first sample after it."""
        t1 = time.perf_counter()
        if self.thread is not None:
            t_end = t1 + 0.1
            while (not any(t > t1 for t, *_ in self.samples) and self.nvml_err is None
                   and time.perf_counter() < t_end):
                time.sleep(0.001)
        self.stop_flag = True
        if self.thread is not None:
            self.thread.join(timeout=5)
        smi = self._smi()
        inside = [x for x in self.samples if self.t0 <= x[0] <= t1]
        after = [x for x in self.samples if x[0] > t1][:1]
        picked = inside or after
        reasons, sm, smax = set(), [], None
        for _, mhz, mx, rs in picked:
            sm.append(float(mhz))
            smax = float(mx)
            reasons |= {nm for nm, bit in self.REASONS if rs & bit}
        source = "nvml 1 ms" if inside else "nvml, first sample after the region"
        if not sm:
            source = "nvidia-smi 200 ms"
            for mhz, mx, rs in smi:
                sm.append(mhz)
                smax = mx
                reasons |= rs
        else:
            for _, _, rs in smi:
                reasons |= rs
        busy = [v for v in sm if smax and v > 0.3 * smax] or sm
        out = {"sm_mhz": float(np.median(busy)) if busy else None, "sm_max_mhz": smax,
               "reasons": sorted(reasons), "samples": len(sm), "smi_samples": len(smi),
               "source": source}
        if self.nvml_err:
            out["nvml_error"] = self.nvml_err
        return out


def _oracle_threads(n):
    """Set the oracle's OpenMP thread count (libgomp, through the oracle's
    own handle); returns the count in effect."""
    import ctypes
    import oracle
    L = oracle.lib()
    try:
        L.omp_set_num_threads(ctypes.c_int(int(n)))
        L.omp_get_max_threads.restype = ctypes.c_int
        return int(L.omp_get_max_threads())
    except AttributeError:
        return oracle.threads()


def cpu_gemm_sample(sample_rows=256, sample_cols=4096, seconds_target=10.0):
    """The oracle, as it stands, on a bounded sample of the prefill workload:
    quantize `sample_rows` rows of A and `sample_cols` rows of W (NVFP4,
    global scales of the sample), dequantize, binary64 GEMM.  Returns
    (TFLOP/s of the sampled GEMM incl. its quantization, threads, description)."""
    import oracle
    from mxfp4_block_scaled_fp4_b200 import inputs
    g = inputs.rng(99, sample_rows, sample_cols, K)
    a = inputs.to_bf16(inputs.normal(g, (sample_rows, K)))
    w = inputs.to_bf16(inputs.normal(g, (sample_cols, K), 0.02))
    oracle.lib()
    reps, t_total = 0, 0.0
    while t_total < seconds_target and reps < 50:
        t0 = time.perf_counter()
        ca, sa, ga = oracle.quantize_nvfp4(a)
        cw, sw, gw = oracle.quantize_nvfp4(w)
        oracle.gemm(oracle.dequant(ca, sa, 0, ga), oracle.dequant(cw, sw, 0, gw))
        t_total += time.perf_counter() - t0
        reps += 1
    flop = 2.0 * sample_rows * sample_cols * K * reps
    desc = (f"{sample_rows} rows of A x {sample_cols} rows of W at K={K} (NVFP4 quantize of "
            f"both + binary64 GEMM), {reps} repetitions, {t_total:.1f} s")
    return flop / t_total / 1e12, oracle.threads(), desc


def cpu_quantize_sweep(all_threads):
    """The oracle's quantizers on the activation-quantize sweep (M in {1, 32,
    512, 8192} x K in {2880, 8192, 16384}; NVFP4 DYNAMIC, NVFP4 STATIC g=0.05,
    MXFP4), in GB/s with the GPU sweep's single-pass byte accounting: every
    shape in full on all cores, and on one core a bounded sample (the shapes
    with M <= 512 in full, the first 64 rows of each M = 8192 shape)."""
    import oracle
    from mxfp4_block_scaled_fp4_b200 import inputs
    variants = (("nvfp4_dynamic", 0, None), ("nvfp4_static", 0, 0.05), ("mxfp4", 1, None))
    data = {(m, k): inputs.act_sweep(m, k) for (m, k) in SWEEP_SHAPES}
    out = {}
    for label, nthreads, row_cap in (("all_cores", all_threads, None), ("one_core", 1, 64)):
        used = _oracle_threads(nthreads)
        res = {}
        for name, fmt, g in variants:
            byts, secs = 0.0, 0.0
            for (m, k), x in data.items():
                xs = x if row_cap is None or m <= 512 else x[:row_cap].contiguous()
                t0 = time.perf_counter()
                oracle.quantize(xs, fmt, g)
                secs += time.perf_counter() - t0
                byts += (2.5625 if fmt == 0 else 2.53125) * xs.shape[0] * k
            res[name] = {"gbs_single_pass": round(byts / secs / 1e9, 4), "seconds": round(secs, 2)}
        res["threads"] = used
        res["sample"] = ("all 12 shapes in full" if row_cap is None else
                         "M <= 512 shapes in full, first 64 rows of each M = 8192 shape")
        out[label] = res
    _oracle_threads(all_threads)
    return out


def cpu_decode_shapes(threads):
    """The oracle on the decode shapes in full (M in {1, 8, 32} x (N, K) in
    {(4096, 4096), (14336, 4096), (4096, 14336)}): per call the activation's
    DYNAMIC NVFP4 quantization, the dequantization of both operands and the
    binary64 GEMM (weights quantized once per shape, untimed, as at load);
    the faster of two calls.  Effective GB/s with the GPU decode rows' byte
    accounting."""
    import oracle
    from mxfp4_block_scaled_fp4_b200 import inputs
    _oracle_threads(threads)
    rows = []
    for (N, Kd) in ((4096, 4096), (14336, 4096), (4096, 14336)):
        _, w = inputs.decode(1, N, Kd)
        cw, sw, gw = oracle.quantize_nvfp4(w)
        for Md in (1, 8, 32):
            a, _ = inputs.decode(Md, N, Kd)
            sec = float("inf")
            for _ in range(2):   # the faster of two calls (the first pays page faults)
                t0 = time.perf_counter()
                ca, sa, ga = oracle.quantize_nvfp4(a)
                oracle.gemm(oracle.dequant(ca, sa, 0, ga), oracle.dequant(cw, sw, 0, gw))
                sec = min(sec, time.perf_counter() - t0)
            rows.append({"M": Md, "N": N, "K": Kd, "us": round(sec * 1e6, 1),
                         "gbs": round(decode_bytes(Md, N, Kd) / sec / 1e9, 4)})
    return rows


def cpu_baseline(full=True):
    """The three legs of the CPU-oracle baseline: the prefill GEMM on a row
    sample (the headline value), the quantize sweep on all cores and one
    core, and the decode shapes in full."""
    val, cores, desc = cpu_gemm_sample()
    out = {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}
    if full:
        out["legs"] = {"quantize_sweep": cpu_quantize_sweep(cores),
                       "decode": cpu_decode_shapes(cores)}
    return out




def flush_l2(torch, buf_w, buf_r):
    """Evict L2: write a buffer twice its size, then read another one, so the
    timed kernel meets clean (not dirty) lines."""
    buf_w.zero_()
    buf_r.sum()


def decode_bytes(M, N, K):
    """Algorithmic bytes of one fused decode call: packed weights + their
    E4M3 scales, the bf16 activation read once, the bf16 output written."""
    return N * K * 0.5625 + M * K * 2 + M * N * 2


def measure_decode(torch, ops, L, inputs, dev, hbm_peak, shapes=None):
    """fp4_gemm_fused on the decode shapes: (i) one call after an L2 flush,
    (ii) back-to-back calls inside one captured CUDA graph, cycling through
    enough weight copies that every call streams its weights from HBM."""
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    out = []
    w_cache = {}
    for (M, N, K) in (shapes or DECODE_SHAPES):
        if (N, K) not in w_cache:
            w_cache.clear()
            _, w = inputs.decode(1, N, K)
            w_cache[(N, K)] = ops.quantize_weights(w.to(dev), L.FP4_NVFP4)
        wq0 = w_cache[(N, K)]
        x = inputs.random_bf16(7, (M, K)).to(dev)
        wbytes = wq0.codes.numel() + wq0.scales.numel()
        copies = max(2, -(-3 * L2_BYTES // wbytes))
        wqs = [ops.Quantized(wq0.codes.clone(), wq0.scales.clone(), wq0.g.clone(), wq0.fmt,
                             wq0.layout, wq0.rows, wq0.K) for _ in range(copies)]
        c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        g_out = torch.empty(1, dtype=torch.float32, device=dev)
        for wq in wqs[:2]:
            ops.gemm_fused(x, wq, out=c, g_out=g_out)
        torch.cuda.synchronize(dev)
        # (i) single call, cold L2
        cold = []
        for i in range(5):
            flush_l2(torch, flush, flush_r)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            ops.gemm_fused(x, wqs[i % copies], out=c, g_out=g_out)
            e1.record()
            torch.cuda.synchronize(dev)
            cold.append(e0.elapsed_time(e1) * 1e3)
        # (ii) graph of `copies` back-to-back calls
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for wq in wqs:
                ops.gemm_fused(x, wq, out=c, g_out=g_out)
        graph.replay()
        torch.cuda.synchronize(dev)
        reps = max(3, int(2000 // copies))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize(dev)
        us = e0.elapsed_time(e1) * 1e3 / (reps * copies)
        gbs = decode_bytes(M, N, K) / (us * 1e-6) / 1e9
        out.append({"M": M, "N": N, "K": K, "us_graph": round(us, 3),
                    "gbs_graph": round(gbs, 1), "frac_hbm": round(gbs / hbm_peak, 4),
                    "us_cold_single": round(float(np.median(cold)), 3),
                    "weight_copies": copies})
        del graph, wqs
    return out


def measure_vendor(torch, ops, a_dev, w_dev, dev, M, N, K):
    """Context only: the vendor library's block-scaled FP4 GEMM (cuBLASLt,
    reached through torch's scaled_mm) on the same quantized operands, bf16
    out, timed like fp4_gemm (L2 flushed before each call).  Not part of the
    product path; reports why if the library call is unavailable."""
    try:
        import torch.nn.functional as F
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        flush_r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        a, w = a_dev, w_dev
        res = {}
        for fmt, name, sdt, rec in ((0, "nvfp4", torch.float8_e4m3fn, F.ScalingType.BlockWise1x16),
                                    (1, "mxfp4", torch.float8_e8m0fnu, F.ScalingType.BlockWise1x32)):
            aq = ops.quantize(a, fmt, ops.SCALES_MMA)
            wq = ops.quantize_weights(w, fmt)
            A = aq.codes.view(torch.float4_e2m1fn_x2)
            B = wq.codes.view(torch.float4_e2m1fn_x2).t()
            sa, sb = aq.scales.view(sdt), wq.scales.view(sdt)
            sw = F.SwizzleType.SWIZZLE_32_4_4
            c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            calls = {"ours": lambda: ops.gemm(aq, wq, out=c),
                     "vendor": lambda: F.scaled_mm(A, B, sa, rec, sb, rec, sw, sw,
                                                   output_dtype=torch.bfloat16)}
            # how far the vendor's result is from ours (it takes no global
            # scales: NVFP4 is rescaled by g_a g_w), relative to ours' rms
            ref = ops.gemm(aq, wq, out=c).float()
            vend = calls["vendor"]().float()
            if fmt == 0:
                vend = vend * (aq.g * wq.g)
            rel = float(((vend - ref).abs().max() / ref.pow(2).mean().sqrt()).item())
            ms = {}
            for key, fn in calls.items():
                for _ in range(3):
                    fn()
                ts = []
                for _ in range(10):
                    flush_l2(torch, flush, flush_r)
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record()
                    fn()
                    e1.record()
                    torch.cuda.synchronize(dev)
                    ts.append(e0.elapsed_time(e1))
                ms[key] = float(np.median(ts))
            fl = 2.0 * M * N * K
            res[name] = {"ours_tflops": round(fl / ms["ours"] / 1e9, 1),
                         "vendor_tflops": round(fl / ms["vendor"] / 1e9, 1),
                         "ours_over_vendor": round(ms["vendor"] / ms["ours"], 3),
                         "vendor_max_diff_over_rms": round(rel, 4)}
        res["vendor"] = "cuBLASLt block-scaled FP4 GEMM via torch.nn.functional.scaled_mm"
        return res
    except Exception as e:  # context only: never fails the bench
        return {"unavailable": f"{type(e).__name__}: {str(e)[:200]}"}


PREFILL_MATRIX = [(2048, 8192), (2048, 28672), (8192, 8192), (8192, 28672)]


def measure_prefill_matrix(torch, L, ops, a_big, w_big, dev, fp4_peak):
    """The prefill GEMM matrix (M in {2048, 8192} x (N, K) in {(8192, 8192),
    (28672, 8192)}; NVFP4 with bf16 and fp32 output, MXFP4 with bf16): per
    row the GEMM alone (operands quantized beforehand) and the step
    quantize_act + GEMM, each timed call after an L2 flush, median of 20.
    Operands are the leading rows of the bench's 8192 x 8192 activation and
    28672 x 8192 weight (same distributions as the prefill recipe)."""
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    sp = torch.cuda.current_stream(dev).cuda_stream
    rows = []

    def timed(fn, reps=20):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            flush_l2(torch, flush, flush_r)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
        return float(np.median(ts))

    for (Mr, Nr) in PREFILL_MATRIX:
        a = a_big[:Mr]
        w = w_big[:Nr]
        flop = 2.0 * Mr * Nr * K
        for fmt in (0, 1):
            wq = ops.quantize_weights(w, fmt)
            aq = ops.quantize(a, fmt, ops.SCALES_MMA)
            ws_bytes = L.fp4_workspace_bytes(Mr, Nr, K, fmt)
            ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
            for out_dt in ((torch.bfloat16, torch.float32) if fmt == 0 else (torch.bfloat16,)):
                c = torch.empty((Mr, Nr), dtype=out_dt, device=dev)
                o = 1 if out_dt == torch.float32 else 0

                def gemm_only():
                    st = L.fp4_gemm(aq.codes.data_ptr(), aq.scales.data_ptr(), aq.g.data_ptr(),
                                    wq.codes.data_ptr(), wq.scales.data_ptr(), wq.g.data_ptr(),
                                    Mr, Nr, K, fmt, c.data_ptr(), Nr, o, None, 0, 0, sp)
                    assert st == 0, st

                def step():
                    st = L.fp4_quantize_act(a.data_ptr(), Mr, K, fmt, 0, 0, aq.g.data_ptr(),
                                            aq.codes.data_ptr(), aq.scales.data_ptr(),
                                            ws.data_ptr(), ws_bytes, sp)
                    assert st == 0, st
                    gemm_only()

                g_ms = timed(gemm_only)
                s_ms = timed(step)
                rows.append({"M": Mr, "N": Nr, "K": K, "format": "NVFP4" if fmt == 0 else "MXFP4",
                             "out": "fp32" if o else "bf16",
                             "gemm_ms": round(g_ms, 4),
                             "gemm_tflops": round(flop / g_ms / 1e9, 1),
                             "gemm_frac_fp4_peak": round(flop / g_ms / 1e9 / fp4_peak, 4),
                             "step_ms": round(s_ms, 4),
                             "step_tflops": round(flop / s_ms / 1e9, 1),
                             "kernel": gemm_kernel_name(Mr, Nr, K)})
                del c
            del wq, aq, ws
    st, code = ops.device_status()
    if st != 0:
        raise RuntimeError(f"status word set in the prefill matrix: {code:#x}")
    return rows


MOE_CONFIGS = [(8, 16384, 4096, 4096), (64, 16384, 2048, 4096)]


def cool_down(torch, dev, seconds=2.0):
    """Lets the GPU idle for a moment between supplementary measurements."""
    torch.cuda.synchronize(dev)
    time.sleep(seconds)


def grouped_kernel_name(M, N, E, sms=148):
    """The kernel fp4_gemm_grouped launches for M routed rows over E groups
    (its launch rule: the CTA-pair form when groups average 512 rows or more
    and its 256 x 256 tiles keep half the SMs busy)."""
    pair_ctas = 2 * (-(-M // 256)) * (-(-N // 256))
    if M >= 512 * E and N > 128 and M > 128 and 2 * pair_ctas >= sms:
        return "fp4 gemm_pair_kernel grouped (256x256 tiles on CTA pairs"
    return ("fp4 gemm_kernel grouped (128x256 tiles" if N > 128 else
            "fp4 gemm_kernel grouped (128x128 tiles")


def measure_grouped(torch, ops, dev, fp4_peak):
    """The grouped (mixture-of-experts) GEMM, fp4_gemm_grouped: E experts of
    [N, K], 16384 routed rows (8192 tokens x 2 experts each) spread over the
    experts with Dirichlet(1) proportions (seed 11; uneven groups that start
    on any row), NVFP4 and MXFP4, bf16 out.  Each call after an L2 flush,
    median of 20.  Also the same work as E separate fp4_gemm calls."""
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    rows = []
    for (E, M, N, Kx) in MOE_CONFIGS:
        rng = np.random.default_rng(11)
        sizes = np.floor(rng.dirichlet(np.ones(E)) * M).astype(np.int64)
        sizes[0] += M - sizes.sum()
        offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
        gen = torch.Generator(device=dev)
        gen.manual_seed(12)
        a = torch.randn((M, Kx), generator=gen, device=dev).to(torch.bfloat16)
        w = (torch.randn((E, N, Kx), generator=gen, device=dev) * 0.02).to(torch.bfloat16)
        offs_d = torch.from_numpy(offs).to(dev)
        flop = 2.0 * M * N * Kx
        for fmt in (0, 1):
            aq = ops.quantize(a, fmt, ops.SCALES_MMA)
            wq = ops.quantize_experts(w, fmt)
            c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            subs = []
            for e in range(E):
                lo, hi = int(offs[e]), int(offs[e + 1])
                if hi > lo:
                    subs.append((lo, hi, ops.quantize(a[lo:hi].contiguous(), fmt, ops.SCALES_MMA,
                                                      g=aq.g if fmt == 0 else None),
                                 ops.Quantized(wq.codes[e], wq.scales[e], wq.g[e:e + 1], fmt,
                                               ops.SCALES_MMA, N, Kx)))

            def grouped():
                ops.gemm_grouped(aq, wq, offs_d, out=c)

            def separate():
                for lo, hi, sq, one in subs:
                    ops.gemm(sq, one, out=c[lo:hi])

            res = {}
            clk = None
            for name, fn in (("grouped", grouped), ("separate_calls", separate)):
                for _ in range(3):
                    fn()
                ts = []
                if name == "grouped":
                    clk = Clocks(dev.index or 0)
                    clk.start()
                for _ in range(20):
                    flush_l2(torch, flush, flush_r)
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record()
                    fn()
                    e1.record()
                    torch.cuda.synchronize(dev)
                    ts.append(e0.elapsed_time(e1))
                if name == "grouped":
                    clk = clk.stop()
                res[name] = float(np.median(ts))
            rows.append({"E": E, "M_routed": M, "N": N, "K": Kx,
                         "sm_mhz_during_grouped": clk.get("sm_mhz"),
                         "throttle_reasons": clk.get("reasons"),
                         "format": "NVFP4" if fmt == 0 else "MXFP4",
                         "group_rows_min_max": [int(sizes.min()), int(sizes.max())],
                         "grouped_ms": round(res["grouped"], 4),
                         "grouped_tflops": round(flop / res["grouped"] / 1e9, 1),
                         "grouped_frac_fp4_peak": round(flop / res["grouped"] / 1e9 / fp4_peak, 4),
                         "separate_calls_ms": round(res["separate_calls"], 4),
                         "kernel": grouped_kernel_name(M, N, E) + ", device-side offsets)"})
    st, code = ops.device_status()
    if st != 0:
        raise RuntimeError(f"status word set in the grouped GEMM: {code:#x}")
    return rows


def measure_gemm_quant(torch, ops, a, w_dev, dev, fp4_peak):
    """The GEMM whose epilogue emits the next layer's FP4 activation
    (fp4_gemm_quant, NVFP4 STATIC g and MXFP4) on the prefill matrix's
    largest shape, against fp4_gemm with bf16 out; each call after an L2
    flush, median of 20."""
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    Mq, Nq = a.shape[0], w_dev.shape[0]
    flop = 2.0 * Mq * Nq * K
    rows = []
    for fmt in (0, 1):
        aq = ops.quantize(a, fmt, ops.SCALES_MMA)
        wq = ops.quantize_weights(w_dev, fmt)
        g_out = torch.tensor([0.004], dtype=torch.float32, device=dev)
        c = torch.empty((Mq, Nq), dtype=torch.bfloat16, device=dev)
        res = {}
        for name, fn in (("bf16_out", lambda: ops.gemm(aq, wq, out=c)),
                         ("fp4_out", lambda: ops.gemm_quant(aq, wq, fmt, ops.SCALES_MMA, g_out))):
            for _ in range(3):
                fn()
            ts = []
            for _ in range(20):
                flush_l2(torch, flush, flush_r)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize(dev)
                ts.append(e0.elapsed_time(e1))
            res[name] = float(np.median(ts))
        out_bytes = Mq * Nq // 2 + Mq * Nq // (16 if fmt == 0 else 32)
        rows.append({"M": Mq, "N": Nq, "K": K, "format": "NVFP4" if fmt == 0 else "MXFP4",
                     "fp4_out_ms": round(res["fp4_out"], 4),
                     "fp4_out_tflops": round(flop / res["fp4_out"] / 1e9, 1),
                     "fp4_out_frac_fp4_peak": round(flop / res["fp4_out"] / 1e9 / fp4_peak, 4),
                     "bf16_out_ms": round(res["bf16_out"], 4),
                     "bytes_written_fp4_vs_bf16": [out_bytes, Mq * Nq * 2]})
    return rows


def measure_mbs(torch, ops, a, w_dev, dev, fp4_peak):
    """MXFP4 with macro-block scaling on the largest prefill shape: the GEMM
    alone (fp4_gemm_mbs) against the plain MXFP4 GEMM, and the activation
    quantizer (row pass + quantize pass) against the plain one; each call
    after an L2 flush, median of 20."""
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    Mq, Nq = a.shape[0], w_dev.shape[0]
    flop = 2.0 * Mq * Nq * K
    aq_m = ops.quantize(a, 1, ops.SCALES_MMA, mbs=True)
    wq_m = ops.quantize_weights(w_dev, 1, mbs=True)
    aq_p = ops.quantize(a, 1, ops.SCALES_MMA)
    wq_p = ops.quantize_weights(w_dev, 1)
    c = torch.empty((Mq, Nq), dtype=torch.bfloat16, device=dev)
    res = {}
    for name, fn in (("gemm_mbs", lambda: ops.gemm(aq_m, wq_m, out=c)),
                     ("gemm_plain", lambda: ops.gemm(aq_p, wq_p, out=c)),
                     ("quantize_mbs", lambda: ops.quantize(a, 1, ops.SCALES_MMA, mbs=True)),
                     ("quantize_plain", lambda: ops.quantize(a, 1, ops.SCALES_MMA))):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(20):
            flush_l2(torch, flush, flush_r)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
        res[name] = float(np.median(ts))
    return {"M": Mq, "N": Nq, "K": K, "format": "MXFP4 + per-row macro scales",
            "gemm_mbs_ms": round(res["gemm_mbs"], 4),
            "gemm_mbs_tflops": round(flop / res["gemm_mbs"] / 1e9, 1),
            "gemm_mbs_frac_fp4_peak": round(flop / res["gemm_mbs"] / 1e9 / fp4_peak, 4),
            "gemm_plain_ms": round(res["gemm_plain"], 4),
            "quantize_mbs_ms": round(res["quantize_mbs"], 4),
            "quantize_plain_ms": round(res["quantize_plain"], 4),
            "note": "quantize_mbs reads the activation twice (row pass + quantize pass)"}


def measure_quantize_sweep(torch, L, inputs, dev, hbm_peak, shapes=None):
    """fp4_quantize_act_ex on the activation-quantize sweep, L2 flushed
    before every call: NVFP4 DYNAMIC / STATIC, MXFP4, and the options (the
    online Hadamard rotation of order 16 / 32, the overflow-aware MXFP4
    rule).  Reports GB/s with single-pass bytes (2.5625 B/elem NVFP4,
    2.53125 MXFP4) and, for the DYNAMIC NVFP4 runs, with both reads of the
    amax pass (4.5625 B/elem)."""
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    sp = torch.cuda.current_stream(dev).cuda_stream
    res = []
    for (M, K) in (shapes or SWEEP_SHAPES):
        x = inputs.act_sweep(M, K).to(dev)
        # context: a plain device copy of the same tensor (2 B read + 2 B
        # written per element), timed the same way -- the bandwidth a tensor
        # of this size reaches at all, fixed costs included
        y = torch.empty_like(x)
        cts = []
        for i in range(8):
            flush_l2(torch, flush, flush_r)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            y.copy_(x)
            e1.record()
            torch.cuda.synchronize(dev)
            if i >= 3:
                cts.append(e0.elapsed_time(e1) * 1e3)
        copy_us = float(np.median(cts))
        copy_gbs = 4.0 * M * K / (copy_us * 1e-6) / 1e9
        del y
        for fmt, gmode, name, had, rule in (
                (0, 0, "nvfp4_dynamic", 0, 0), (0, 1, "nvfp4_static", 0, 0), (1, 0, "mxfp4", 0, 0),
                (0, 0, "nvfp4_dynamic_hadamard16", 16, 0), (1, 0, "mxfp4_hadamard32", 32, 0),
                (1, 0, "mxfp4_oas", 0, 1)):
            opt = L.opts(had, rule)
            codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
            scales = torch.empty(L.fp4_scale_bytes(M, K, fmt, 0), dtype=torch.uint8, device=dev)
            g = torch.full((1,), 0.05, dtype=torch.float32, device=dev)
            wsb = L.fp4_workspace_bytes(M, 0, K, fmt)
            ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
            ts = []
            for i in range(8):
                flush_l2(torch, flush, flush_r)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                st = L.fp4_quantize_act_ex(x.data_ptr(), M, K, fmt, 0, gmode, opt, g.data_ptr(),
                                           codes.data_ptr(), scales.data_ptr(), ws.data_ptr(),
                                           wsb, sp)
                e1.record()
                torch.cuda.synchronize(dev)
                assert st == 0
                if i >= 3:
                    ts.append(e0.elapsed_time(e1) * 1e3)
            us = float(np.median(ts))
            single = (2.5625 if fmt == 0 else 2.53125) * M * K
            row = {"M": M, "K": K, "variant": name, "us": round(us, 3),
                   "gbs_single_pass": round(single / (us * 1e-6) / 1e9, 1)}
            if gmode == 0 and fmt == 0:
                two = 4.5625 * M * K
                row["gbs_two_reads"] = round(two / (us * 1e-6) / 1e9, 1)
                row["frac_hbm_two_reads"] = round(two / (us * 1e-6) / 1e9 / hbm_peak, 4)
            row["frac_hbm_single_pass"] = round(single / (us * 1e-6) / 1e9 / hbm_peak, 4)
            row["same_size_copy_gbs"] = round(copy_gbs, 1)
            # a copy moves 4 B per element, this pass 2.5 - 4.6: at sizes
            # where fixed costs dominate both take about the same time
            row["same_size_copy_us"] = round(copy_us, 3)
            row["copy_us_over_pass_us"] = round(copy_us / us, 3)
            res.append(row)
    return res


def measure_decoder(torch, dev, batch_sizes=(1, 16, 256), reps=20):
    """The synthetic 24-layer decoder (288 W4A4 GEMM calls per forward) and
    the same forward in torch bf16, each captured once as a CUDA graph."""
    from mxfp4_block_scaled_fp4_b200.decoder import SyntheticDecoder
    dec = SyntheticDecoder(dev)
    res = []
    for M in batch_sizes:
        x = torch.randn(M, 2880, generator=torch.Generator().manual_seed(M)).to(torch.bfloat16).to(dev)
        row = {"M": M, "gemm_calls": 288}
        for name, fn in (("fp4", dec.forward_fp4), ("bf16", dec.forward_bf16)):
            g, _ = dec.capture(fn, x)
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize(dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
            torch.cuda.synchronize(dev)
            row[f"us_per_forward_{name}"] = round(e0.elapsed_time(e1) * 1e3 / reps, 1)
            del g
        row["speedup_vs_bf16"] = round(row["us_per_forward_bf16"] / row["us_per_forward_fp4"], 3)
        row["fp4_weight_bytes"] = dec.weight_bytes()
        row["structure"] = ("per layer q|k|v, o, gate0|gate1|up0|up1, down0..3 as concurrent "
                            "graph branches; bf16: q|k|v, o, gate|up, down")
        res.append(row)
    return res


def max_over_ranks(torch, values, device):
    """Element-wise maximum of per-rank timings over all ranks of the process
    group (the job's time is its slowest replica's); the values unchanged on
    a single process."""
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tflops(flop_per_rank, world, ms):
    """Whole-job throughput: every rank runs one replica of the step."""
    return flop_per_rank * world / (ms * 1e-3) / 1e12


def run_part(args, rank):
    """One supplementary measurement alone (profiling aid)."""
    import torch
    from mxfp4_block_scaled_fp4_b200 import fp4lib as L, inputs, ops
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    L.lib()
    peaks, _ = load_peaks()
    line = {"metric": METRIC, "impl": "ours", "part": args.only}
    if args.only == "decode":
        shapes = None
        if args.decode_shape:
            shapes = [tuple(int(v) for v in args.decode_shape.split(","))]
        line["decode"] = measure_decode(torch, ops, L, inputs, dev, peaks["hbm_gbs"], shapes)
    elif args.only == "decoder":
        line["decoder"] = measure_decoder(torch, dev)
    elif args.only == "grouped":
        peaks_fp4 = peaks["bf16_tflops"] * FP4_OVER_BF16
        line["grouped"] = measure_grouped(torch, ops, dev, peaks_fp4)
    else:
        shapes = None
        if args.quant_shape:
            shapes = [tuple(int(v) for v in args.quant_shape.split(","))]
        line["quantize_sweep"] = measure_quantize_sweep(torch, L, inputs, dev, peaks["hbm_gbs"],
                                                        shapes)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_reference(args, rank):
    if rank != 0:
        return 0
    val, cores, desc = cpu_gemm_sample(
        seconds_target=min(20.0, max(5.0, 0.5 * (args.steps + args.warmup))))
    line = {
        "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": FLOP / (val * 1e12) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "sample": desc},
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-suite", action="store_true",
                    help="skip the decode and quantize-sweep measurements")
    ap.add_argument("--only", default="all",
                    choices=["all", "prefill", "decode", "quantize", "decoder", "grouped"],
                    help="run one part only (profiling); the JSON line then carries that part")
    ap.add_argument("--decode-shape", default=None, help="M,N,K: restrict the decode part")
    ap.add_argument("--quant-shape", default=None, help="M,K: restrict the quantize part")
    ap.add_argument("--shape", default=None,
                    help="M,N,K override (profiling of smaller cases); default 8192,28672,8192")
    args = ap.parse_args()
    if args.shape:
        global M, N, K, FLOP, WORKLOAD
        M, N, K = (int(v) for v in args.shape.split(","))
        FLOP = 2.0 * M * N * K
        WORKLOAD = (f"W4A4 NVFP4 GEMM M={M} N={N} K={K}, bf16 out, activation quantized per step"
                    " (profiling shape)")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    if args.only in ("decode", "quantize", "decoder", "grouped"):
        return run_part(args, rank)
    if args.warmup < 3:
        args.warmup = 3

    import torch
    import torch.distributed as dist
    from mxfp4_block_scaled_fp4_b200 import fp4lib as L, inputs, ops

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    L.lib()

    a_cpu, w_cpu = inputs.prefill(M, N, K)
    a = a_cpu.to(dev)
    w_dev = w_cpu.to(dev)
    wq = ops.quantize_weights(w_dev, L.FP4_NVFP4)   # load-time step, untimed
    del w_cpu
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(L.fp4_scale_bytes(M, K, 0, 0), dtype=torch.uint8, device=dev)
    g_a = torch.empty(1, dtype=torch.float32, device=dev)
    c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws_bytes = L.fp4_workspace_bytes(M, N, K, 0)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def check(st, what):
        if st != 0:
            raise L.Fp4Error(st, what)

    ev_q0, ev_q1, ev_g1 = ([torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
                           for _ in range(3))

    def step(i=None, timed=False):
        if timed:
            ev_q0[i].record(stream)
        check(L.fp4_quantize_act(a.data_ptr(), M, K, 0, 0, 0, g_a.data_ptr(), codes.data_ptr(),
                                 scales.data_ptr(), ws.data_ptr(), ws_bytes, sp), "quantize")
        if timed:
            ev_q1[i].record(stream)
        check(L.fp4_gemm(codes.data_ptr(), scales.data_ptr(), g_a.data_ptr(), wq.codes.data_ptr(),
                         wq.scales.data_ptr(), wq.g.data_ptr(), M, N, K, 0, c.data_ptr(), N, 0,
                         ws.data_ptr(), ws_bytes, 0, sp), "gemm")
        if timed:
            ev_g1[i].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st, code = ops.device_status()
    if st != 0:
        raise RuntimeError(f"watchdog raised during warm-up: {code:#x}")

    clocks = Clocks(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(i, timed=True)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    ms_total = t_start.elapsed_time(t_end)
    q_ms = float(np.mean([ev_q0[i].elapsed_time(ev_q1[i]) for i in range(args.steps)]))
    g_ms = float(np.mean([ev_q1[i].elapsed_time(ev_g1[i]) for i in range(args.steps)]))
    st, code = ops.device_status()
    if st != 0:
        raise RuntimeError(f"watchdog raised during timing: {code:#x}")

    # ---- end to end through the C ABI with host buffers (pinned).  Every step
    # copies its input from the host and reads its result back; successive
    # steps are pipelined the way a caller would run them: two buffer sets
    # and three streams, so step i's compute overlaps step i+1's upload and
    # step i-1's read-back (PCIe is full duplex).
    a_host = a_cpu.pin_memory()
    c_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    bufs = [dict(a=a, c=c, codes=codes, scales=scales, g=g_a, ws=ws),
            dict(a=torch.empty_like(a), c=torch.empty_like(c), codes=torch.empty_like(codes),
                 scales=torch.empty_like(scales), g=torch.empty_like(g_a),
                 ws=torch.empty_like(ws))]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in, ev_done, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_step(i):
        b = bufs[i % 2]
        if i >= 2:
            s_in.wait_event(ev_done[i % 2])            # this input buffer's last step is done
        with torch.cuda.stream(s_in):
            b["a"].copy_(a_host, non_blocking=True)
        ev_in[i % 2].record(s_in)
        s_comp.wait_event(ev_in[i % 2])
        if i >= 2:
            s_comp.wait_event(ev_out[i % 2])           # this output buffer has been read back
        cs = s_comp.cuda_stream
        check(L.fp4_quantize_act(b["a"].data_ptr(), M, K, 0, 0, 0, b["g"].data_ptr(),
                                 b["codes"].data_ptr(), b["scales"].data_ptr(), b["ws"].data_ptr(),
                                 ws_bytes, cs), "quantize")
        check(L.fp4_gemm(b["codes"].data_ptr(), b["scales"].data_ptr(), b["g"].data_ptr(),
                         wq.codes.data_ptr(), wq.scales.data_ptr(), wq.g.data_ptr(), M, N, K, 0,
                         b["c"].data_ptr(), N, 0, b["ws"].data_ptr(), ws_bytes, 0, cs), "gemm")
        ev_done[i % 2].record(s_comp)
        s_out.wait_event(ev_done[i % 2])
        with torch.cuda.stream(s_out):
            c_host.copy_(b["c"], non_blocking=True)
        ev_out[i % 2].record(s_out)

    e_steps = max(4, min(args.steps, 8))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(e_steps):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e_steps

    ms_total, e2e_ms, g_ms, q_ms = max_over_ranks(torch, [ms_total, e2e_ms, g_ms, q_ms], dev)
    ms_step = ms_total / args.steps

    peaks, src = load_peaks()
    # The timed region is short (milliseconds to a second), so the GEMM is
    # held against the burst bf16 figure x the nominal FP4/BF16 ratio; the
    # nominal dense FP4 peak and a peak scaled to the region's median SM clock
    # are reported beside it.
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    gemm_tflops = FLOP / (g_ms * 1e-3) / 1e12
    q_bytes = QUANT_BYTES_PER_ELEM * M * K
    q_gbs = q_bytes / (q_ms * 1e-3) / 1e9
    sm_mhz, sm_max = clk.get("sm_mhz"), clk.get("sm_max_mhz") or peaks.get("sm_max_mhz")
    roofline = {"bound": "tensor", "achieved": gemm_tflops, "peak": fp4_peak,
                "unit": "TFLOP/s", "frac": gemm_tflops / fp4_peak,
                "traffic": GEMM_TRAFFIC_BYTES if (M, N, K) == (8192, 28672, 8192) else None,
                "traffic_unit": "bytes per launch (ncu dram__bytes_read + write)",
                "kernel": gemm_kernel_name(M, N, K),
                "peak_source": (f"{src} bf16_tflops (burst) x {FP4_OVER_BF16:g} (nominal dense "
                                "FP4/BF16 ratio); of measured"),
                "frac_of_nominal_fp4": gemm_tflops / FP4_NOMINAL_TFLOPS,
                "nominal_fp4_tflops": FP4_NOMINAL_TFLOPS}
    if sm_mhz and sm_max:
        roofline["peak_at_region_clock"] = fp4_peak * sm_mhz / sm_max
        roofline["frac_at_region_clock"] = gemm_tflops / roofline["peak_at_region_clock"]
        roofline["gemm_ms_x_sm_mhz"] = g_ms * sm_mhz

    line = {
        "metric": METRIC,
        "value": job_tflops(FLOP, world, ms_step),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e4m3 scales, fp32 accumulate, bf16 out)",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K, "format": "NVFP4",
                   "global_scale": "dynamic", "out": "bf16",
                   "parallelism": f"replicas x{world}",
                   "l2": (f"{'inputs larger than L2' if M * K * 2 > L2_BYTES else 'A fits in L2'} "
                          f"(A {M * K * 2 >> 20} MiB, packed W {N * K // 2 >> 20} MiB, "
                          f"C {M * N * 2 >> 20} MiB)")},
        "roofline": roofline,
        "quantize": {"achieved_gbs": q_gbs, "peak_gbs": peaks["hbm_gbs"],
                     "frac": q_gbs / peaks["hbm_gbs"], "ms": q_ms,
                     "bytes_per_elem": QUANT_BYTES_PER_ELEM,
                     "note": "amax pass + quantize pass, algorithmic bytes (two reads of A)"},
        "gemm_ms": g_ms,
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
        "e2e": {"value": job_tflops(FLOP, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": a_host.numel() * 2, "d2h_bytes_per_step": c_host.numel() * 2},
    }
    if not args.no_suite and (M, N, K) == (8192, 28672, 8192):
        # each supplementary part starts after a short idle, so that the
        # 1 kW power cap that the previous part's seconds of dense GEMMs
        # engage has released (the grouped rows record their clocks)
        line["prefill_matrix"] = measure_prefill_matrix(torch, L, ops, a, w_dev, dev, fp4_peak)
        cool_down(torch, dev)
        line["gemm_quant"] = measure_gemm_quant(torch, ops, a, w_dev, dev, fp4_peak)
        cool_down(torch, dev)
        line["grouped"] = measure_grouped(torch, ops, dev, fp4_peak)
        cool_down(torch, dev)
        line["mbs"] = measure_mbs(torch, ops, a, w_dev, dev, fp4_peak)
    if not args.no_suite:
        line["decode"] = measure_decode(torch, ops, L, inputs, dev, peaks["hbm_gbs"])
        line["quantize_sweep"] = measure_quantize_sweep(torch, L, inputs, dev, peaks["hbm_gbs"])
        line["decoder"] = measure_decoder(torch, dev)
        line["vendor_reference"] = measure_vendor(torch, ops, a, w_dev, dev, M, N, K)
        line["gpu_launches_note"] = ("gpu_launches counts the timed prefill steps only; the "
                                     "decode and sweep objects are timed separately")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(full=not args.no_suite)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
