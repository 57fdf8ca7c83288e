#!/usr/bin/env python
"""Benchmark of the block-scaled microscaling hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the MXFP4 routed-expert workload: quantize bf16
weights [8, 2048, 7168] to packed e2m1 + e8m0 scales, dequantize packed
weights back to bf16 and to fp32 (three kernels).  Inputs (235 MB) and outputs
are larger than the 126 MB L2, and the dequantize kernels read packed buffers
written two steps earlier (three rotating slots), so every byte is an HBM byte.
`value` is algorithmic bytes (each input read once, each output written once)
per second over the timed region, summed over ranks (weak scaling: each rank
runs its own copy of the workload; the path has no data exchange).

The same run also times the other workloads as sub-measurements ("extra"):
NVFP4 [256, 2048] round trip latency, MXFP8 quantize / dequantize of the
same [8, 2048, 7168] expert weights, the list-of-blocks NVFP4 KV-cache
dequantize (1024 blocks of 64 tokens x 8 heads), the cache fake-quant cases, the
[7168, 18432] NVFP4 weight quantization (ModelOpt per-tensor, per-row,
gate/up, the static two-level fake-quant) and the fused-dequant grouped GEMM
(TFLOP/s), each with its HBM or tensor roofline.

--impl reference times the CPU oracle (the only reference this path has) on a
bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quant/dequant GB/s (% HBM peak); dequant grouped-GEMM TFLOP/s (% bf16 peak)"
E, N, K = 8, 2048, 7168
# GPU spin (about 100 us at 1.9 GHz) queued in front of a timed launch
HOST_COVER_CYCLES = 200_000
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="skip the sub-measurements of the other workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    ap.add_argument("--only", default="", help="run only these sub-measurements (comma list of nvfp4,mxfp8,kv,"
                    "cache,linear,gemm; linear_tensor, linear_row, linear_gu, linear_dq, linear_static pick one row "
                    "of linear) and print them, without the main step; for profiling")
    ap.add_argument("--gemm-only", default="", help="time only these grouped-GEMM variants (comma list of "
                    "mxfp4_fwd,mxfp4_bwd,nvfp4_fwd,nvfp4_bwd,skew) and print them; for profiling")
    return ap.parse_args()


def load_peaks():
    """The measured denominators from MEASURED_PEAKS.json, each key falling
    back to FALLBACK_PEAKS when absent or not a positive number (a value may
    be a number or an object with a "value")."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            raw = json.load(f)
    except Exception:
        return dict(FALLBACK_PEAKS, sources={k: "fallback" for k in FALLBACK_PEAKS}), "fallback"
    peaks, measured = dict(FALLBACK_PEAKS), False
    sources = {k: "fallback" for k in FALLBACK_PEAKS}
    for k in FALLBACK_PEAKS:
        v = raw.get(k) if isinstance(raw, dict) else None
        if isinstance(v, dict):
            v = v.get("value")
        try:
            v = float(v)
        except (TypeError, ValueError):
            continue
        if v > 0:
            peaks[k] = v
            sources[k] = "measured"
            measured = measured or k == "hbm_gbs"
    peaks["sources"] = sources
    return peaks, ("measured" if measured else "fallback")


KERNEL_SOURCES = {
    "flat": ["flat.cu", "common.cuh", "formats.cuh", "host_util.h", "debug.cuh"],
    "nvfp4": ["nvfp4.cu", "common.cuh", "formats.cuh", "host_util.h", "debug.cuh"],
    "cache": ["cache.cu", "common.cuh", "formats.cuh", "host_util.h", "debug.cuh"],
    "static": ["static.cu", "common.cuh", "formats.cuh", "host_util.h", "debug.cuh"],
    "kv": ["kv_cache.cu", "common.cuh", "formats.cuh", "host_util.h", "debug.cuh"],
    "gemm": ["grouped_mm.cu", "tcgen05.cuh", "formats.cuh", "host_util.h", "debug.cuh"],
}


_COMMENT = re.compile(r"//[^\n]*|/\*.*?\*/", re.S)


def kernel_source_hash(family):
    """Hash of the source files a kernel family is built from, with C/C++
    comments and whitespace runs left out, so that a documentation edit does
    not retire a committed ncu traffic figure but any change to the code does
    (the figure is only reported while the hash matches)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fp8_microscaling_quantization_b200", "csrc")
    for name in KERNEL_SOURCES[family]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            code = " ".join(_COMMENT.sub(" ", f.read()).split())
        h.update(name.encode())
        h.update(code.encode())
    return h.hexdigest()[:16]


def traffic_from_profiles(*kernel_keys):
    """Per-launch DRAM bytes (read + write, summed over the given kernels) from
    the committed ncu summary profiles/dram_traffic.json, or None if an entry
    is missing or was taken on other sources than the kernel family's current
    ones."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    total = 0
    for key in kernel_keys:
        ent = d.get("kernels", {}).get(key)
        if not ent or ent.get("family") not in KERNEL_SOURCES:
            return None
        if ent.get("source_hash") != kernel_source_hash(ent["family"]):
            return None
        total += ent.get("bytes_per_launch", 0)
    return total


# ------------------------------------------------------------ multi-rank --

def job_time_ms(dist, region_ms, device):
    """The job's time for the timed region: the maximum over ranks (each rank
    times its own region with CUDA events; the slowest one ends the job)."""
    import torch
    t = torch.tensor([float(region_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world, step_bytes, ms_per_step):
    """Whole-job throughput in GB/s: every rank runs its own copy of the
    workload (weak scaling), so the job moves world * step_bytes per step."""
    return world * step_bytes / (ms_per_step * 1e-3) / 1e9


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        def reader():
            for line in self.proc.stdout:
                self.samples.append((time.time(), [s.strip() for s in line.split(",")]))
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        if self.proc is None:
            return {"unavailable": "nvidia-smi not runnable"}
        sel = [s for t, s in self.samples if t0 <= t <= t1 and len(s) >= 9]
        if not sel:
            sel = [s for t, s in self.samples if len(s) >= 9][-5:]
        if not sel:
            return {"unavailable": "no samples"}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = sorted(v for v in (num(s[1]) for s in sel) if v is not None)
        mx = max((v for v in (num(s[2]) for s in sel) if v is not None), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in sel for i in range(4) if s[5 + i].lower().startswith("active")})
        pw = [v for v in (num(s[3]) for s in sel) if v is not None]
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(sel), "power_w_max": max(pw) if pw else None}


# ------------------------------------------------------------------- utils --

def mx_bytes():
    n = E * N * K
    q = 2 * n + n // 2 + n // 32
    dq_b = n // 2 + n // 32 + 2 * n
    dq_f = n // 2 + n // 32 + 4 * n
    return q, dq_b, dq_f


class Timer:
    """CUDA-event timing of individual launches on the launching stream."""

    def __init__(self, torch, stream):
        self.torch = torch
        self.stream = stream
        self.pending = {}

    def run(self, key, fn):
        ev0 = self.torch.cuda.Event(enable_timing=True)
        ev1 = self.torch.cuda.Event(enable_timing=True)
        ev0.record(self.stream)
        fn()
        ev1.record(self.stream)
        self.pending.setdefault(key, []).append((ev0, ev1))

    def avg_ms(self, key):
        evs = self.pending.get(key, [])
        if not evs:
            return None
        return sum(a.elapsed_time(b) for a, b in evs) / len(evs)


def l2_flush(torch, buf):
    """Evict the L2 by reading a buffer twice its size (a read leaves clean
    lines behind, so no write-back competes with the kernel timed next)."""
    buf.max()


# ------------------------------------------------------- CPU oracle baseline -
#
# The CPU oracle, as it stands (plain scalar C called through ctypes), timed on
# the host cores.  ctypes releases the GIL for the length of each C call, so
# host threads that each run the oracle on their own slice of rows run in
# parallel; nothing in the oracle is changed or tuned for this.  Every row of
# the path gets two figures: one thread, and one thread per core of
# os.sched_getaffinity.  Samples are whole rows (or cache blocks) of the same
# workloads, sized to a fraction of a second per figure; the rate is bytes (or
# FLOPs) per second, so a sample and the full tensor share the unit.

def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _run_parts(fn, parts, threads):
    """Wall seconds to run fn(part) for every part on `threads` host threads."""
    from concurrent.futures import ThreadPoolExecutor
    t0 = time.perf_counter()
    if threads <= 1:
        for part in parts:
            fn(part)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fn, parts))
    return time.perf_counter() - t0


def _split_rows(a, n):
    """n contiguous row slices of a (views; the oracle needs no copy)."""
    import numpy as np
    edges = np.linspace(0, a.shape[0], n + 1).astype(int)
    return [a[edges[i]:edges[i + 1]] for i in range(n) if edges[i + 1] > edges[i]]


class OracleCase:
    """One row of the path for the CPU oracle: make(rows) builds a seeded input
    of `rows` rows (untimed), run(part) processes a row slice of it,
    bytes_per_row is the row's algorithmic bytes (as on the GPU)."""

    def __init__(self, make, run, bytes_per_row, full_rows, split=None):
        self.make, self.run, self.bytes_per_row, self.full_rows = make, run, bytes_per_row, full_rows
        self.split = split or _split_rows


def time_oracle_case(case, cores, seconds=0.4, probe_rows=8):
    """Single-thread and all-core rates of one case, in GB/s, on samples sized
    to about `seconds` each (never more rows than the full workload)."""
    probe = case.make(probe_rows)
    t = max(_run_parts(case.run, [probe], 1), 1e-4)
    rows1 = int(max(probe_rows, min(case.full_rows, probe_rows * seconds / t)))
    x1 = case.make(rows1)
    t1 = _run_parts(case.run, [x1], 1)
    del x1
    rows_n = int(max(rows1, min(case.full_rows, rows1 * cores)))
    xn = case.make(rows_n)
    parts = case.split(xn, cores)
    tn = _run_parts(case.run, parts, cores)
    b1, bn = rows1 * case.bytes_per_row, rows_n * case.bytes_per_row
    return {"single_thread": {"GB/s": round(b1 / t1 / 1e9, 4), "rows": rows1, "s": round(t1, 3)},
            "all_cores": {"GB/s": round(bn / tn / 1e9, 4), "rows": rows_n, "s": round(tn, 3), "threads": len(parts)},
            "full_rows": case.full_rows}


def mx_round_trip_case():
    """The bench step's workload: MXFP4 quantize + dequantize to bf16 and fp32,
    rows of 7168 from the [8*2048, 7168] expert weights."""
    import oracle
    from fp8_microscaling_quantization_b200 import synth

    def make(rows):
        return synth.expert_weights(E=1, N=rows, K=K, zero_blocks=min(4, rows * K // 32), seed=20260002).reshape(rows, K)

    def run(x):
        pk, sc = oracle.quantize_mxfp4(x)
        oracle.dequantize_mxfp4(pk, sc, out_dtype=oracle.BF16)
        oracle.dequantize_mxfp4(pk, sc, out_dtype=oracle.F32)

    q, d1, d2 = mx_bytes()
    return OracleCase(make, run, (q + d1 + d2) // (E * N), E * N)


def oracle_cases():
    """The CPU oracle's counterpart of every sub-measurement, keyed as in the
    GPU output: {(section, row): OracleCase}."""
    import numpy as np
    import oracle
    from fp8_microscaling_quantization_b200 import synth
    cases = {}

    # NVFP4 [256, 2048], per-row scale: quantize; dequantize to bf16
    Kn = 2048
    nb = 2 * Kn + Kn // 2 + Kn // 16 + 4
    cases[("nvfp4_256x2048", "quantize")] = OracleCase(
        lambda r: synth.nvfp4_matrix(rows=r, cols=Kn, seed=20260001), lambda x: oracle.quantize_nvfp4(x), nb, 256)

    def make_nv_q(rows, cols=Kn, seed=20260001):
        # dequantize inputs: random packed codes, finite e4m3 scales, row scales
        rng = np.random.default_rng(seed)
        return (rng.integers(0, 256, (rows, cols // 2), dtype=np.uint8),
                rng.integers(0, 0x7F, (rows, cols // 16), dtype=np.uint8),
                (rng.random(rows) * 1e-3).astype(np.float32))

    def split3(t, n):
        pk, sc, g = t
        return list(zip(_split_rows(pk, n), _split_rows(sc, n), _split_rows(g, n)))

    cases[("nvfp4_256x2048", "dequantize_bf16")] = OracleCase(
        make_nv_q, lambda t: oracle.dequantize_nvfp4(*t, out_dtype=oracle.BF16), nb, 256, split3)

    # MXFP8 on the [8, 2048, 7168] expert weights
    def make_w(rows):
        return synth.expert_weights(E=1, N=rows, K=K, zero_blocks=min(4, rows * K // 32), seed=20260006).reshape(rows, K)

    def split2(t, n):
        return list(zip(_split_rows(t[0], n), _split_rows(t[1], n)))

    cases[("mxfp8_expert_weights_8x2048x7168", "quantize")] = OracleCase(
        make_w, lambda x: oracle.quantize_mxfp8(x), 2 * K + K + K // 32, E * N)
    def make_mx8_codes(rows):
        rng = np.random.default_rng(20260006)
        c = rng.integers(0, 0x7F, (rows, K), dtype=np.uint8) | (rng.integers(0, 2, (rows, K), dtype=np.uint8) << 7)
        return (c, rng.integers(100, 130, (rows, K // 32), dtype=np.uint8))

    cases[("mxfp8_expert_weights_8x2048x7168", "dequantize_bf16")] = OracleCase(
        make_mx8_codes, lambda t: oracle.dequantize_mxfp8(*t, out_dtype=oracle.BF16), K + K // 32 + 2 * K, E * N,
        split2)

    # the FP8 stored form (power-of-two scale per 32-block) on the same weights
    cases[("fp8_pow2_expert_weights_8x2048x7168", "quantize")] = OracleCase(
        make_w, lambda x: oracle.quantize_fp8(x, 32), 2 * K + K + K // 32, E * N)
    cases[("fp8_pow2_expert_weights_8x2048x7168", "dequantize_bf16")] = OracleCase(
        make_mx8_codes, lambda t: oracle.dequantize_fp8(t[0], t[1], 32, out_dtype=oracle.BF16), K + K // 32 + 2 * K,
        E * N, split2)

    # KV cache: a "row" is one block of 64 tokens x 8 heads x 128
    bt, hd = 64, 8
    rows_kv = bt * hd

    def make_kv(nblk):
        rng = np.random.default_rng(20260007)
        vals = [rng.integers(0, 256, (rows_kv, 64), dtype=np.uint8) for _ in range(nblk)]
        scs = [rng.integers(0, 0x7E, (rows_kv, 8), dtype=np.uint8) for _ in range(nblk)]
        am = (rng.random(nblk) * 100).astype(np.float32)
        return (vals, scs, am)

    def split_kv(t, n):
        vals, scs, am = t
        edges = np.linspace(0, len(vals), n + 1).astype(int)
        return [(vals[a:b], scs[a:b], am[a:b]) for a, b in zip(edges[:-1], edges[1:]) if b > a]

    nkv = rows_kv * 128
    cases[("kv_cache_nvfp4_1024x64x8x128", "dequantize_bf16")] = OracleCase(
        make_kv, lambda t: oracle.dequantize_kv_cache_nvfp4(t[0], t[1], t[2], bt, hd), nkv // 2 + nkv // 16 + 4 + 2 * nkv,
        1024, split_kv)

    # quantize_cache: a row is one [C] vector of the [B, T, C] activations
    for name, fmt, blk, (Bc, Tc, C) in (
            ("fp8_b32_4x8192x512", 0, 32, (4, 8192, 512)), ("mxfp4_b32_4x8192x128", 1, 32, (4, 8192, 128)),
            ("nvfp4_b16_4x2048x512", 2, 16, (4, 2048, 512)), ("fp8_b32_4x2048x520", 0, 32, (4, 2048, 520)),
            ("mxfp4_b32_4x2048x520", 1, 32, (4, 2048, 520)), ("nvfp4_b16_4x2048x520", 2, 16, (4, 2048, 520))):
        cases[("quantize_cache", name)] = OracleCase(
            (lambda C: lambda r: synth.cache_acts(B=1, T=r, C=C, seed=20260003)[0].reshape(r, C))(C),
            (lambda fmt, blk: lambda x: oracle.quantize_cache(x, fmt, blk))(fmt, blk), 4 * C, Bc * Tc)
    cases[("quantize_cache", "ste_backward_copy_4x8192x512")] = OracleCase(
        lambda r: synth.cache_acts(B=1, T=r, C=512, seed=20260003)[1].reshape(r, 512),
        lambda g: oracle.quantize_cache_backward(g), 4 * 512, 4 * 8192)

    # [7168, 18432] linear weight
    Kl = 18432
    nrow = 2 * Kl + Kl // 2 + Kl // 16

    def make_lin(r):
        return synth.linear_weight(out=r, inp=Kl, seed=20260004)

    sec = "nvfp4_linear_7168x18432"
    # per-tensor: each thread quantizes its own slice with that slice's tensor
    # scale (the same work per element as one tensor scale over all rows)
    cases[(sec, "modelopt_tensor_scale")] = OracleCase(make_lin, lambda x: oracle.quantize_nvfp4_tensor(x),
                                                       nrow + 2 * Kl, 7168)
    cases[(sec, "per_row_scale")] = OracleCase(make_lin, lambda x: oracle.quantize_nvfp4(x), nrow + 4, 7168)

    def make_gu(r):
        x = make_lin(r)
        return (x, np.full(r, 1e-5, np.float32))

    cases[(sec, "gate_up_given_row_scales_14336x18432")] = OracleCase(
        make_gu, lambda t: oracle.quantize_nvfp4(t[0], row_scale=t[1]), nrow + 8, 14336, split2)
    cases[(sec, "dequantize_bf16")] = OracleCase(
        lambda r: make_nv_q(r, Kl, 20260004), lambda t: oracle.dequantize_nvfp4(*t, out_dtype=oracle.BF16),
        Kl // 2 + Kl // 16 + 4 + 2 * Kl, 7168, split3)

    def make_static(r):
        x = make_lin(r)
        xf = synth.bf16_bits_to_f32(x)
        bam = np.abs(xf).reshape(r, -1, 16).max(axis=2).astype(np.float32)
        return (x, bam, float(np.abs(xf).max()))

    def split_static(t, n):
        return [(a, b, t[2]) for a, b in zip(_split_rows(t[0], n), _split_rows(t[1], n))]

    cases[(sec, "static_two_level_fake_quant")] = OracleCase(
        make_static, lambda t: oracle.fake_quantize_nvfp4_static(*t), 2 * Kl + 4 * (Kl // 16) + 2 * Kl, 7168,
        split_static)
    return cases


def time_oracle_gemm(cores, offs):
    """The grouped GEMM's CPU reference (the oracle's binary32 dequantization of
    each expert, then a float64 library matmul), timed on one expert with a
    sample of rows and extrapolated linearly to the full problem: 32 expert
    dequantizations plus T rows of products.  The matmul uses the BLAS threads
    of numpy (one, then `cores`)."""
    import numpy as np
    import oracle
    from threadpoolctl import threadpool_limits
    from fp8_microscaling_quantization_b200 import synth
    T, Kd, Nd, Ed = 16384, 7168, 2048, 32
    rows = 256
    rng = np.random.default_rng(20260005)
    w = synth.to_bf16_bits((rng.standard_normal((Nd, Kd), dtype=np.float32) * np.float32(0.02)))
    pk, sc = oracle.quantize_mxfp4(w)
    a = synth.to_bf16_bits(rng.standard_normal((rows, Kd), dtype=np.float32))
    del w
    out = {}
    for label, threads in (("single_thread", 1), ("all_cores", cores)):
        with threadpool_limits(limits=threads):
            t0 = time.perf_counter()
            W = oracle.dequant_expert_f32(oracle.FMT_MXFP4, pk, sc).astype(np.float64)
            t_dq = time.perf_counter() - t0
            A = oracle.bf16_to_f32(a).astype(np.float64)
            t0 = time.perf_counter()
            _ = A @ W.T
            t_mm = time.perf_counter() - t0
        t_full = Ed * t_dq + T / rows * t_mm
        out[label] = {"TFLOP/s": round(2.0 * T * Nd * Kd / t_full / 1e12, 6), "s_full_extrapolated": round(t_full, 2),
                      "threads": threads}
    out["sample"] = (f"MXFP4 forward: one expert [2048, 7168] dequantized by the oracle, then {rows} rows of the "
                     f"float64 product; extrapolated to 32 experts and T=16384 (extrapolated)")
    return out


def run_cpu_oracle_rows(cores):
    """CPU oracle figures for every sub-measurement: {section: {row: {...}}}."""
    res = {}
    for (sec, row), case in oracle_cases().items():
        try:
            t0 = time.perf_counter()
            res.setdefault(sec, {})[row] = time_oracle_case(case, cores)
            res[sec][row]["wall_s"] = round(time.perf_counter() - t0, 2)
        except Exception as ex:  # report, never hide
            res.setdefault(sec, {})[row] = {"unavailable": f"{type(ex).__name__}: {ex}"}
    try:
        res["grouped_gemm"] = {"mxfp4_fwd": time_oracle_gemm(cores, None)}
    except Exception as ex:
        res["grouped_gemm"] = {"unavailable": f"{type(ex).__name__}: {ex}"}
    return res


def run_cpu_baseline():
    """The bench step's workload on the CPU oracle: all cores (the reported
    value) and one thread."""
    cores = host_cores()
    r = time_oracle_case(mx_round_trip_case(), cores, seconds=2.0)
    mt, st = r["all_cores"], r["single_thread"]
    return {"value": mt["GB/s"], "unit": "GB/s", "cores": mt["threads"], "kind": "oracle",
            "single_thread": {"value": st["GB/s"], "cores": 1, "rows": st["rows"], "s": st["s"]},
            "sample": f"{mt['rows']} rows x 7168 of the MXFP4 expert-weight workload (quantize + dequantize bf16 + "
                      f"dequantize fp32), C oracle on {mt['threads']} host threads, {mt['s']} s; single thread: "
                      f"{st['rows']} rows, {st['s']} s"}


def merge_oracle_rows(extra, oracle_rows):
    """Put each CPU-oracle figure beside its GPU row as "oracle_cpu"."""
    for sec, rows in oracle_rows.items():
        dst = extra.setdefault(sec, {})
        if not isinstance(dst, dict):
            continue
        if sec == "grouped_gemm":
            dst["oracle_cpu"] = rows
            continue
        for row, fig in rows.items():
            ent = dst.setdefault(row, {})
            if isinstance(ent, dict):
                ent["oracle_cpu"] = fig


# --------------------------------------------------------------- reference --

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    steps, warmup = max(1, args.steps), max(0, args.warmup)
    cores = host_cores()
    case = mx_round_trip_case()
    rows = 256 * cores  # 256 rows per host thread per step
    x = case.make(rows)
    parts = case.split(x, cores)
    for _ in range(warmup):
        _run_parts(case.run, parts, cores)
    tot_t, done = 0.0, 0
    t_start = time.perf_counter()
    for _ in range(steps):
        tot_t += _run_parts(case.run, parts, cores)
        done += 1
        if time.perf_counter() - t_start > 150:
            break
    val = done * rows * case.bytes_per_row / tot_t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": done, "warmup": warmup, "ms_per_step": round(tot_t / done * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "mxfp4_expert_weights_round_trip", "shape": [E, N, K],
                       "sample_rows_per_step": rows},
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": len(parts), "kind": "oracle",
                             "sample": f"{rows} rows x 7168 per step (quantize + dequantize bf16 + fp32) on "
                                       f"{len(parts)} host threads"},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- ours ---

def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    if args.gemm_only:
        from fp8_microscaling_quantization_b200 import bsq, synth
        peaks, peak_kind = load_peaks()
        dev = torch.device("cuda", 0)
        res = bench_gemm(torch, bsq, synth, dev, torch.cuda.current_stream(), peaks, peak_kind,
                         variants=set(args.gemm_only.split(",")), iters=max(1, args.steps), warm=args.warmup)
        print(json.dumps({"grouped_gemm": res}), flush=True)
        return
    if args.only:
        from fp8_microscaling_quantization_b200 import bsq, synth
        peaks, peak_kind = load_peaks()
        dev = torch.device("cuda", 0)
        res = run_extra(torch, bsq, synth, dev, torch.cuda.current_stream(), peaks, peak_kind,
                        set(filter(None, args.only.split(","))))
        print(json.dumps({"extra": res}), flush=True)
        return
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    from fp8_microscaling_quantization_b200 import bsq, synth

    peaks, peak_kind = load_peaks()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    steps, warmup = max(1, args.steps), max(3, args.warmup)

    # ---- workload: MXFP4 routed-expert weights [8, 2048, 7168] --------------
    g = torch.Generator(device=dev)
    g.manual_seed(20260002 + rank)
    xs = [synth.expert_weights_torch(E, N, K, generator=g, device=dev) for _ in range(2)]
    packed = [torch.empty((E, N, K // 2), dtype=torch.uint8, device=dev) for _ in range(3)]
    scales = [torch.empty((E, N, K // 32), dtype=torch.uint8, device=dev) for _ in range(3)]
    yb = torch.empty((E, N, K), dtype=torch.bfloat16, device=dev)
    yf = torch.empty((E, N, K), dtype=torch.float32, device=dev)
    for i in range(3):
        bsq.bsq_quantize_mxfp4(xs[i % 2], packed=packed[i], scales=scales[i])
    torch.cuda.synchronize()

    timer = Timer(torch, stream)

    def step(i, timed):
        q = lambda: bsq.bsq_quantize_mxfp4(xs[i % 2], packed=packed[i % 3], scales=scales[i % 3])
        d1 = lambda: bsq.bsq_dequantize_mxfp4(packed[(i + 1) % 3], scales[(i + 1) % 3], y=yb)
        d2 = lambda: bsq.bsq_dequantize_mxfp4(packed[(i + 2) % 3], scales[(i + 2) % 3], y=yf)
        if timed:
            timer.run("mx_quant", q)
            timer.run("mx_dequant_bf16", d1)
            timer.run("mx_dequant_fp32", d2)
        else:
            q(), d1(), d2()

    for i in range(warmup):
        step(i, False)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    t_soak = time.time()
    i = 0
    while time.time() - t_soak < 1.0:  # keep the GPU under this load while clocks settle
        step(i, False)
        i += 1
        if i % 50 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev_start = torch.cuda.Event(enable_timing=True)
    ev_end = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    ev_start.record(stream)
    for i in range(steps):
        step(i, True)
    ev_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    clocks.stop()
    region_ms = ev_start.elapsed_time(ev_end)
    if world > 1:
        region_ms = job_time_ms(dist, region_ms, dev)
    ms_per_step = region_ms / steps
    qb, db, fb = mx_bytes()
    step_bytes = qb + db + fb
    value = job_value(world, step_bytes, ms_per_step)

    kern = {}
    for key, nbytes in (("mx_quant", qb), ("mx_dequant_bf16", db), ("mx_dequant_fp32", fb)):
        ms = timer.avg_ms(key)
        kern[key] = {"ms": round(ms, 5), "bytes": nbytes, "GB/s": round(nbytes / ms / 1e6, 1),
                     "frac_hbm": round(nbytes / ms / 1e6 / peaks["hbm_gbs"], 4)}
    dom = max(kern, key=lambda k: kern[k]["ms"])
    roof = {"kernel": dom, "bound": "hbm", "achieved": kern[dom]["GB/s"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": kern[dom]["frac_hbm"], "traffic": traffic_from_profiles(dom),
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback"}

    # ---- end to end through the public API with pinned host buffers ---------
    e2e = None
    if rank == 0 or world > 1:
        e2e = measure_e2e(torch, bsq, xs[0], stream, steps=min(steps, 10))

    line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": steps,
            "warmup": warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "mxfp4_expert_weights_round_trip: bf16 [8,2048,7168] -> int8 packed + e8m0 "
                                   "-> bf16 and fp32", "l2": "inputs and outputs larger than L2; dequantize reads "
                                   "packed buffers from 3 rotating slots", "parallelism": f"replicas x{world}",
                       "frac_hbm_step": round(value / world / peaks["hbm_gbs"], 4)},
            "roofline": roof, "kernels": kern, "gpu_launches": 3 * steps,
            "clocks": clocks.summary(t_soak, t_wall1)}
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and rank == 0 and not args.no_cpu:
        try:
            line["cpu_baseline"] = run_cpu_baseline()
        except Exception as ex:  # report, never hide
            line["cpu_baseline"] = {"unavailable": f"{type(ex).__name__}: {ex}"}
    if not args.no_extra and world == 1:
        line["extra"] = run_extra(torch, bsq, synth, dev, stream, peaks, peak_kind, set())
        if rank == 0 and not args.no_cpu:
            merge_oracle_rows(line["extra"], run_cpu_oracle_rows(host_cores()))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def measure_e2e(torch, bsq, x_dev, stream, steps):
    """Quantize + dequantize through the C ABI with the step's input copied from
    pinned host memory and every output copied back, inside the timed region.
    Steps are pipelined over two buffer slots: step i's outputs stream back on
    a copy stream while step i + 1's input streams in and its kernels run, so
    the two PCIe directions overlap (the host-to-device copy, the kernels and
    the device-to-host copy of every step are all inside the region)."""
    xh = x_dev.cpu().pin_memory()
    dev = x_dev.device
    xd = [torch.empty_like(x_dev) for _ in range(2)]
    p = [torch.empty((E, N, K // 2), dtype=torch.uint8, device=dev) for _ in range(2)]
    s = [torch.empty((E, N, K // 32), dtype=torch.uint8, device=dev) for _ in range(2)]
    yb = [torch.empty((E, N, K), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    yf = [torch.empty((E, N, K), dtype=torch.float32, device=dev) for _ in range(2)]
    ph = [torch.empty_like(p[0], device="cpu").pin_memory() for _ in range(2)]
    sh = [torch.empty_like(s[0], device="cpu").pin_memory() for _ in range(2)]
    ybh = [torch.empty_like(yb[0], device="cpu").pin_memory() for _ in range(2)]
    yfh = [torch.empty_like(yf[0], device="cpu").pin_memory() for _ in range(2)]
    out_stream = torch.cuda.Stream(device=dev)
    computed = [torch.cuda.Event() for _ in range(2)]
    drained = [torch.cuda.Event() for _ in range(2)]

    def step(i):
        k = i % 2
        if i >= 2:
            stream.wait_event(drained[k])  # slot k's previous outputs are on the host
        with torch.cuda.stream(stream):
            xd[k].copy_(xh, non_blocking=True)
            bsq.bsq_quantize_mxfp4(xd[k], packed=p[k], scales=s[k])
            bsq.bsq_dequantize_mxfp4(p[k], s[k], y=yb[k])
            bsq.bsq_dequantize_mxfp4(p[k], s[k], y=yf[k], out_dtype=bsq.DType.FP32)
        computed[k].record(stream)
        out_stream.wait_event(computed[k])
        with torch.cuda.stream(out_stream):
            ph[k].copy_(p[k], non_blocking=True)
            sh[k].copy_(s[k], non_blocking=True)
            ybh[k].copy_(yb[k], non_blocking=True)
            yfh[k].copy_(yf[k], non_blocking=True)
        drained[k].record(out_stream)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    out_stream.wait_event(e0)
    for i in range(steps):
        step(i)
    out_stream.wait_stream(stream)
    e1.record(out_stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    qb, db, fb = mx_bytes()
    h2d = xh.numel() * 2
    d2h = ph[0].numel() + sh[0].numel() + ybh[0].numel() * 2 + yfh[0].numel() * 4
    return {"value": round((qb + db + fb) / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3),
            "note": "pinned host buffers; two slots, input copy + kernels on one stream, output copy on another"}


# ------------------------------------------------------------- sub-measures -

def run_extra(torch, bsq, synth, dev, stream, peaks, peak_kind, only):
    out = {}
    flush = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    hbm = peaks["hbm_gbs"]

    def timed(fn, iters, cold):
        t = Timer(torch, stream)
        for _ in range(3):
            fn()
        for _ in range(iters):
            if cold:
                l2_flush(torch, flush)
            # keep the GPU busy while the host enqueues the start event and the
            # launch, so the event pair brackets the kernel and not host time
            torch.cuda._sleep(HOST_COVER_CYCLES)
            t.run("k", fn)
        torch.cuda.synchronize()
        return t.avg_ms("k")

    def graph_timed(calls, reps=7):
        """Per-launch ms of `calls` (one launch each) captured into one CUDA
        graph and replayed: the median over `reps` replays of the replay time
        over len(calls).  The launches run back to back with no host gap."""
        for c in calls:  # eager once: fills the library's host-side caches
            c()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for c in calls:
                c()
        graph.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(reps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        del graph
        times.sort()
        return times[len(times) // 2] / len(calls)

    def rec(ms, nbytes, *traffic_keys):
        r = {"us": round(ms * 1e3, 2), "bytes": nbytes, "GB/s": round(nbytes / ms / 1e6, 1),
             "frac_hbm": round(nbytes / ms / 1e6 / hbm, 4)}
        if traffic_keys:
            r["traffic"] = traffic_from_profiles(*traffic_keys)
        return r

    want = (lambda s: not only or s in only)

    if want("nvfp4"):
        g = torch.Generator(device=dev)
        g.manual_seed(20260001)
        x = synth.nvfp4_matrix_torch(256, 2048, generator=g, device=dev)
        p, s, r = bsq.bsq_quantize_nvfp4(x)
        y = torch.empty_like(x)
        n = x.numel()
        nb = 2 * n + n // 2 + n // 16 + 4 * 256
        q_ms = timed(lambda: bsq.bsq_quantize_nvfp4(x, packed=p, scales=s, row_scale_out=r), 50, True)
        d_ms = timed(lambda: bsq.bsq_dequantize_nvfp4(p, s, r, y=y), 50, True)
        # the latency floor at this size: a device-to-device copy of the
        # input, timed the same way (the quantize reads it and writes a
        # quarter of it; the dequantize the reverse)
        c_ms = timed(lambda: y.copy_(x), 50, True)
        qr, dr = rec(q_ms, nb), rec(d_ms, nb)
        for rr, ms in ((qr, q_ms), (dr, d_ms)):
            rr["same_size_copy_us"] = round(c_ms * 1e3, 2)
            rr["frac_of_copy"] = round(c_ms / ms, 4)
        out["nvfp4_256x2048"] = {"quantize": qr, "dequantize_bf16": dr,
                                 "note": "latency-bound (1.3 MB); L2 flushed before every launch"}

    if want("mxfp8"):
        g = torch.Generator(device=dev)
        g.manual_seed(20260006)
        x = synth.expert_weights_torch(E, N, K, generator=g, device=dev)
        n = x.numel()
        c = torch.empty((E, N, K), dtype=torch.uint8, device=dev)
        s = torch.empty((E, N, K // 32), dtype=torch.uint8, device=dev)
        y = torch.empty_like(x)
        out["mxfp8_expert_weights_8x2048x7168"] = {
            "quantize": rec(timed(lambda: bsq.bsq_quantize_mxfp8(x, codes=c, scales=s), 10, False),
                            2 * n + n + n // 32, "mxfp8_quant"),
            "dequantize_bf16": rec(timed(lambda: bsq.bsq_dequantize_mxfp8(c, s, y=y), 10, False),
                                   n + n // 32 + 2 * n, "mxfp8_dequant_bf16"),
            "note": "inputs and outputs larger than L2"}
        # the FP8 stored form (e4m3 codes, power-of-two scale per 32-block) on
        # the same weights: the same kernels with the power-of-two scale rule
        out["fp8_pow2_expert_weights_8x2048x7168"] = {
            "quantize": rec(timed(lambda: bsq.bsq_quantize_fp8(x, 32, codes=c, scales=s), 10, False),
                            2 * n + n + n // 32),
            "dequantize_bf16": rec(timed(lambda: bsq.bsq_dequantize_fp8(c, s, 32, y=y), 10, False),
                                   n + n // 32 + 2 * n),
            "note": "inputs and outputs larger than L2"}
        del x, c, s, y

    if want("kv"):
        g = torch.Generator(device=dev)
        g.manual_seed(20260007)
        nbk, bt, hd = 1024, 64, 8
        rows = bt * hd
        # separate, non-contiguous blocks: views into three allocations with a
        # gap after every block (three launches to fill instead of thousands)
        vpool = torch.randint(0, 256, (nbk, rows + 16, 64), generator=g, device=dev, dtype=torch.uint8)
        spool = torch.randint(0, 0x7E, (nbk, rows + 16, 8), generator=g, device=dev, dtype=torch.uint8)
        apool = torch.rand((nbk, 4), generator=g, device=dev) * 100
        vals = [vpool[i, :rows] for i in range(nbk)]
        scs = [spool[i, :rows] for i in range(nbk)]
        ams = [apool[i, :1] for i in range(nbk)]
        table = bsq.kv_block_table(vals, scs, ams)
        yk = torch.empty((1, nbk * bt, hd, 128), dtype=torch.bfloat16, device=dev)
        n = nbk * rows * 128
        out["kv_cache_nvfp4_1024x64x8x128"] = {
            "dequantize_bf16": rec(timed(lambda: bsq.bsq_dequantize_kv_cache_nvfp4(table, nbk, bt, hd, y=yk), 10, True),
                                   n // 2 + n // 16 + 4 * nbk + 2 * n, "kv_dequant_bf16"),
            "note": "1024 non-contiguous blocks of 64 tokens x 8 heads x 128; L2 flushed before every launch"}
        del vals, scs, ams, vpool, spool, apool, table, yk

    if want("cache"):
        g = torch.Generator(device=dev)
        g.manual_seed(20260003)
        l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
        cases = [("fp8_b32_4x8192x512", 0, 32, (4, 8192, 512)), ("mxfp4_b32_4x8192x128", 1, 32, (4, 8192, 128)),
                 ("nvfp4_b16_4x2048x512", 2, 16, (4, 2048, 512)), ("fp8_b32_4x2048x520", 0, 32, (4, 2048, 520)),
                 ("mxfp4_b32_4x2048x520", 1, 32, (4, 2048, 520)), ("nvfp4_b16_4x2048x520", 2, 16, (4, 2048, 520))]
        res = {}
        for name, fmt, blk, shp in cases:
            x = synth.cache_acts_torch(*shp, generator=g, device=dev)
            y = torch.empty_like(x)
            nb = 2 * 2 * x.numel()
            res[name] = rec(timed(lambda: bsq.bsq_quantize_cache(x, fmt, blk, y=y), 30, True), nb, "cache_" + name)
            # the latency floor at this size: a device-to-device copy of the
            # same bytes, timed the same way
            copy_ms = timed(lambda: y.copy_(x), 30, True)
            res[name]["same_size_copy_us"] = round(copy_ms * 1e3, 2)
            res[name]["frac_of_copy"] = round(copy_ms * 1e3 / res[name]["us"], 4)
            # throughput of back-to-back launches replayed from a CUDA graph,
            # cycling over input/output copies that together exceed twice the
            # L2, so that every launch reads and writes HBM; the same-size copy
            # the same way
            ns = max(2, -(-2 * l2_bytes // nb))
            xs = [x.clone() for _ in range(ns)]
            ys = [torch.empty_like(x) for _ in range(ns)]
            n_calls = max(60, ns)
            g_ms = graph_timed([(lambda i=i: bsq.bsq_quantize_cache(xs[i % ns], fmt, blk, y=ys[i % ns]))
                                for i in range(n_calls)])
            gc_ms = graph_timed([(lambda i=i: ys[i % ns].copy_(xs[i % ns])) for i in range(n_calls)])
            res[name].update({"graph_us": round(g_ms * 1e3, 2), "graph_GB/s": round(nb / g_ms / 1e6, 1),
                              "graph_frac_hbm": round(nb / g_ms / 1e6 / hbm, 4),
                              "graph_copy_us": round(gc_ms * 1e3, 2), "graph_frac_of_copy": round(gc_ms / g_ms, 4),
                              "graph_slots": ns, "graph_launches": n_calls})
            del xs, ys
        gsrc = torch.randn((4, 8192, 512), generator=g, device=dev).to(torch.bfloat16)
        gdst = torch.empty_like(gsrc)
        res["ste_backward_aliased"] = {"us": 0.0, "bytes": 0, "note": "identity: no launch"}
        res["ste_backward_copy_4x8192x512"] = rec(
            timed(lambda: bsq.bsq_quantize_cache_backward(gsrc, gdst), 30, True), 2 * 2 * gsrc.numel())
        res["note"] = ("us: one launch, L2 flushed before it (tensors of 8-34 MB); graph_us: per launch, median "
                       "of 7 replays of a CUDA graph of graph_launches back-to-back launches cycling over "
                       "graph_slots input/output copies that total at least twice the L2")
        out["quantize_cache"] = res

    linear_rows = ("tensor", "row", "gu", "dq", "static")
    want_linear = [r for r in linear_rows if want("linear") or f"linear_{r}" in only]
    if want_linear:
        g = torch.Generator(device=dev)
        g.manual_seed(20260004)
        x = synth.linear_weight_torch(7168, 18432, generator=g, device=dev)
        up = synth.linear_weight_torch(7168, 18432, generator=g, device=dev)
        cat = torch.cat([x, up], 0) if "gu" in want_linear else None
        del up
        n = x.numel()
        p = torch.empty((7168, 18432 // 2), dtype=torch.uint8, device=dev)
        s = torch.empty((7168, 18432 // 16), dtype=torch.uint8, device=dev)
        r = torch.empty((7168,), dtype=torch.float32, device=dev)
        t = torch.empty((1,), dtype=torch.float32, device=dev)
        scratch = torch.empty((bsq.bsq_nvfp4_tensor_scratch_bytes(7168, 18432),), dtype=torch.uint8, device=dev)
        pc = torch.empty((2 * 7168, 18432 // 2), dtype=torch.uint8, device=dev)
        sc = torch.empty((2 * 7168, 18432 // 16), dtype=torch.uint8, device=dev)
        rc = torch.full((2 * 7168,), 1e-5, dtype=torch.float32, device=dev)
        rco = torch.empty_like(rc)
        nb_row = 2 * n + n // 2 + n // 16 + 4 * 7168
        nb_tensor = 4 * n + n // 2 + n // 16 + 4
        nb_gu = 2 * (2 * n) + (2 * n) // 2 + (2 * n) // 16 + 2 * 4 * 14336
        y = torch.empty((7168, 18432), dtype=torch.bfloat16, device=dev)
        nb_dq = n // 2 + n // 16 + 4 * 7168 + 2 * n
        # static two-level fake-quant: calibrated block amax = the data's own
        bam = x.view(-1, 16).abs().amax(dim=1).float()
        gam = x.abs().amax().float().reshape(1)
        nb_st = 2 * n + 4 * (n // 16) + 2 * n
        lin = {}
        if "tensor" in want_linear:
            lin["modelopt_tensor_scale"] = rec(timed(lambda: bsq.bsq_quantize_nvfp4_tensor(
                x, packed=p, scales=s, tensor_scale=t, scratch=scratch), 10, False), nb_tensor,
                "nvfp4_tensor_amax_pass", "nvfp4_tensor_quant_pass")
        if "row" in want_linear:
            lin["per_row_scale"] = rec(timed(lambda: bsq.bsq_quantize_nvfp4(x, packed=p, scales=s, row_scale_out=r),
                                             10, False), nb_row, "nvfp4_per_row")
        if "gu" in want_linear:
            lin["gate_up_given_row_scales_14336x18432"] = rec(timed(lambda: bsq.bsq_quantize_nvfp4(
                cat, row_scale_in=rc, packed=pc, scales=sc, row_scale_out=rco), 10, False), nb_gu,
                "nvfp4_gate_up_given_row_scales")
        if "dq" in want_linear:
            bsq.bsq_quantize_nvfp4(x, packed=p, scales=s, row_scale_out=r)
            lin["dequantize_bf16"] = rec(timed(lambda: bsq.bsq_dequantize_nvfp4(p, s, r, y=y), 10, False), nb_dq,
                                         "nvfp4_dequant_bf16")
        if "static" in want_linear:
            lin["static_two_level_fake_quant"] = rec(timed(
                lambda: bsq.bsq_fake_quantize_nvfp4_static(x, bam, gam, y=y), 10, False), nb_st,
                "nvfp4_static_fake_quant")
        lin["note"] = "inputs larger than L2; per-tensor counts two reads of the input"
        out["nvfp4_linear_7168x18432"] = lin
        del x, cat, y

    if want("gemm"):
        try:
            out["grouped_gemm"] = bench_gemm(torch, bsq, synth, dev, stream, peaks, peak_kind)
        except bsq.BsqError as e:
            out["grouped_gemm"] = {"unavailable": str(e)}
    return out


def bench_gemm(torch, bsq, synth, dev, stream, peaks, peak_kind, variants=None, iters=10, warm=3):
    import numpy as np
    T, Kd, Nd, Ed = 16384, 7168, 2048, 32
    rng = np.random.default_rng(20260005)
    offs_np = synth.zipf_offs(rng, T, Ed)
    g = torch.Generator(device=dev)
    g.manual_seed(20260005)
    x = torch.randn((T, Kd), generator=g, device=dev).to(torch.bfloat16)
    go = torch.randn((T, Nd), generator=g, device=dev).to(torch.bfloat16)
    w = (torch.randn((Ed, Nd, Kd), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    want_mx = not variants or any(v.startswith("mxfp4") or v == "skew" for v in variants)
    want_nv = not variants or any(v.startswith("nvfp4") for v in variants)
    mx_p, mx_s = bsq.bsq_quantize_mxfp4(w) if want_mx else (None, None)
    nv_p, nv_s, nv_r = bsq.bsq_quantize_nvfp4(w) if want_nv else (None, None, None)
    del w
    offs = torch.from_numpy(offs_np).to(dev)
    flops = 2.0 * T * Nd * Kd
    out_f = torch.empty((T, Nd), dtype=torch.bfloat16, device=dev)
    out_b = torch.empty((T, Kd), dtype=torch.bfloat16, device=dev)
    err = torch.zeros((1,), dtype=torch.int32, device=dev)
    res = {"flop_per_launch": flops, "offs": offs_np.tolist()}
    peak = peaks["bf16_tflops"]
    for fmt_name, fmt, p, s, r in (("mxfp4", bsq.Format.MXFP4, mx_p, mx_s, None),
                                   ("nvfp4", bsq.Format.NVFP4, nv_p, nv_s, nv_r)):
        for dname, d, a, o in (("fwd", bsq.Direction.FWD, x, out_f), ("bwd", bsq.Direction.BWD, go, out_b)):
            if variants and f"{fmt_name}_{dname}" not in variants:
                continue
            fn = lambda: bsq.bsq_grouped_mm_fp4(fmt, d, a, p, s, r, offs, out=o, err=err)
            t = Timer(torch, stream)
            for _ in range(warm):
                fn()
            for _ in range(iters):
                t.run("k", fn)
            torch.cuda.synchronize()
            ms = t.avg_ms("k")
            tf = flops / (ms * 1e-3) / 1e12
            res[f"{fmt_name}_{dname}"] = {"us": round(ms * 1e3, 1), "TFLOP/s": round(tf, 1),
                                          "frac_bf16": round(tf / peak, 4),
                                          "traffic": traffic_from_profiles(f"gemm_{fmt_name}_{dname}")}
    # routing skews (MXFP4 forward, same weights and activations): how the
    # 16-token padding of short experts and the tile dealing hold up
    if not variants or "skew" in variants:
        skew = {}
        for kind in ("uniform", "zipf", "hot", "tiny"):
            o_np = synth.skew_offs(np.random.default_rng(20260008), kind, T, Ed)
            o = torch.from_numpy(o_np).to(dev)
            fn = lambda: bsq.bsq_grouped_mm_fp4(bsq.Format.MXFP4, bsq.Direction.FWD, x, mx_p, mx_s, None, o,
                                                out=out_f, err=err)
            t = Timer(torch, stream)
            for _ in range(warm):
                fn()
            for _ in range(iters):
                t.run("k", fn)
            torch.cuda.synchronize()
            ms = t.avg_ms("k")
            tf = flops / (ms * 1e-3) / 1e12
            cnt = np.diff(np.concatenate([[0], o_np]))
            skew[kind] = {"us": round(ms * 1e3, 1), "TFLOP/s": round(tf, 1), "frac_bf16": round(tf / peak, 4),
                          "max_expert_tokens": int(cnt.max()), "experts_under_17_tokens": int((cnt < 17).sum())}
        skew["note"] = "MXFP4 forward, T=16384 K=7168 N=2048 E=32; routing: uniform, Zipf(1.1), one expert with " \
                       "half the tokens, half the experts with 1-16 tokens"
        res["routing_skew_mxfp4_fwd"] = skew
    res["err_word"] = int(err.item())
    res["peak"] = f"{peak} TFLOP/s bf16 dense ({peaks.get('sources', {}).get('bf16_tflops', peak_kind)}, burst)"
    return res


if __name__ == "__main__":
    main()
