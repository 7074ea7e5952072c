#!/usr/bin/env python
"""Benchmark of the W4A16 decode GEMV: microseconds per linear and achieved
HBM bandwidth at M = 1 on the 8192 x 28672 (N x K) Llama-70B-shaped linear
(asymmetric uint4, G = 128, fp16 scale and zero), one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one decode linear y = x dequant(Wq)^T through wq_gemv_w4a16 with the
quantized weights resident in HBM.  Quantization and relayout are the offline
part of the path (done once per model); they run and are timed in the same
process and reported under "offline".  The timed region replays CUDA graphs of
back-to-back GEMV launches that cycle through several copies of the packed
weight (more bytes than L2 holds), bracketed by CUDA events on the launching
stream, with a barrier and a device synchronize on both sides; with N > 1
every rank runs its own replica and the slowest rank's time counts.

--impl reference times the CPU oracle (the plain C restatement of the method)
on the host cores instead, one output row per step, scaled to a full linear.
"""
from __future__ import annotations

import argparse
import csv
import datetime as dt
import hashlib
import re
import io
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W4A16 G128 GEMV µs/linear and achieved HBM TB/s vs B200 peak at M=1"
UNIT = "us/linear"
WORKLOAD_CID, WORKLOAD_LIN = 3, 3          # Llama-70B-shaped linear, N=8192, K=28672
FALLBACK_HBM_GBS = 6650.0
START_DELAY_CYCLES = 500_000                # ~0.25 ms of SM clock ahead of the start event

# DRAM bytes per GEMV launch from an ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum) and the hash of the kernel sources (code only,
# comments removed) it was taken on;
# reported only while the sources are unchanged.
NCU_TRAFFIC = {"sources_sha256": "10e1d16873f7fe3f44f4b7ebdefe2a62826ba7efe2948561dd2b7651b67cea0b",
               "bytes_per_launch": 124883456 + 3779328}


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the offline and other-M legs")
    ap.add_argument("--case", choices=["gemv_m1", "gemv_m4", "gemm_m16", "gemm_m64", "gemm_m512",
                                       "nvfp4_m1", "nvfp4_m128"], default=None,
                    help="run one small profiling case (3 launches) and exit")
    return ap.parse_args()


def algorithmic_bytes(M: int, N: int, K: int, sym: bool) -> int:
    """Bytes the method must move for one linear: packed codes, fp16 scales,
    fp16 zeros (asymmetric), bf16 x and fp32 y."""
    return N * K // 2 + 2 * N * K // 128 + (0 if sym else 2 * N * K // 128) + 2 * M * K + 4 * M * N


def _code_only(src: str) -> str:
    """The source with comments and blank lines removed, so that the hash
    changes with the code and not with its comments."""
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def kernel_sources_sha() -> str:
    h = hashlib.sha256()
    for f in ("wq_gemv.cu", "wq_common.cuh"):
        with open(os.path.join(ROOT, "post_weight_quantization_wq_b200", "csrc", f)) as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "MEASURED_PEAKS.json hbm_gbs (copy bandwidth, measured)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (earlier measurement on this pool)"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons, kept only while
    the timed region runs (by wall-clock timestamp)."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid: str):
        self.uuid = gpu_uuid
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def mark_begin(self):
        self.t0 = dt.datetime.now()

    def mark_end(self):
        self.t1 = dt.datetime.now()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for rec in csv.reader(io.StringIO(out)):
            if len(rec) < 9:
                continue
            rec = [r.strip() for r in rec]
            try:
                ts = dt.datetime.strptime(rec[0], "%Y/%m/%d %H:%M:%S.%f")
            except ValueError:
                continue
            if self.t0 and self.t1 and not (self.t0 <= ts <= self.t1):
                continue
            rows.append(rec)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for rec in rows for n, v in zip(names, rec[5:9]) if v == "Active"})
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": sm[len(sm) // 2] if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(pw) if pw else None,
                "samples": len(rows), "reasons": reasons}


# ------------------------------------------------------------------ our arm

def run_ours(a, rank: int, world: int, local_rank: int):
    import numpy as np
    import torch
    import post_weight_quantization_wq_b200 as wq
    from post_weight_quantization_wq_b200 import _binding as abi
    from post_weight_quantization_wq_b200 import inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    wl = inputs.WORKLOADS[WORKLOAD_CID]
    lin = wl.linears[WORKLOAD_LIN]
    N, K, M, sym = lin.N, lin.K, 1, wl.sym

    W = inputs.workload_weight(WORKLOAD_CID, WORKLOAD_LIN)
    x = inputs.workload_activations(WORKLOAD_CID, WORKLOAD_LIN, M)
    Wt = torch.from_numpy(W.view(np.int16)).to(dev).view(torch.bfloat16)
    xt = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)

    extras = {}
    with torch.cuda.stream(stream):
        qw = wq.quantize(Wt, symmetric=sym, stream=stream)
        if not a.no_extras:
            extras["offline"] = time_offline(Wt, qw, stream, N, K, sym)
    torch.cuda.synchronize(dev)
    del Wt

    # L2 hygiene: cycle through copies of the packed weight, more bytes than L2.
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    wbytes = qw.packed.numel()
    ncopies = max(3, math.ceil(3 * l2 / wbytes))
    copies = [qw.packed] + [qw.packed.clone() for _ in range(ncopies - 1)]
    ws_bytes = abi.wq_workspace_bytes(M, N, K)
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    y = torch.empty((M, N), dtype=torch.float32, device=dev)

    def launch(i, s):
        st = abi.wq_gemv_w4a16(xt, None, copies[i % ncopies], M, N, K, 128, sym, 1, y, ws,
                               ws_bytes, s)
        if st != 0:
            raise wq.WqError(st, "wq_gemv_w4a16")

    chunk = 100 * ncopies
    graphs = build_graphs(launch, stream, a.steps, chunk, dev)

    # warm-up (untimed)
    with torch.cuda.stream(stream):
        for i in range(a.warmup):
            launch(i, stream)
    torch.cuda.synchronize(dev)
    if abi.wq_last_device_status(stream) != 0:
        raise RuntimeError("device error during warm-up")

    sampler = None
    if rank == 0:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
        sampler.start()
    if sampler:
        sampler.mark_begin()
    # Clock window: nvidia-smi samples every 100 ms, longer than a short timed
    # region, so the same graph replays run for about a second right before
    # it (untimed) and the clock record covers both.
    soak = soak_graph(launch, stream, chunk, dev)
    t_soak = time.perf_counter()
    with torch.cuda.stream(stream):
        while time.perf_counter() - t_soak < 1.2:
            soak.replay()
            torch.cuda.synchronize(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):          # graph replays go to the current stream
        # A device-side delay ahead of the start event: the host has submitted
        # the timed graphs by the time the stream reaches e0, so the region
        # measures the launches, not the host's submission latency.
        torch.cuda._sleep(START_DELAY_CYCLES)
        e0.record(stream)
        for g in graphs:
            g.replay()
        e1.record(stream)
    e1.synchronize()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.mark_end()
    barrier(world)
    elapsed_ms = e0.elapsed_time(e1)
    clocks = sampler.stop() if sampler else None
    st = abi.wq_last_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status after timing: {abi.status_string(st)}")
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    if clocks is not None:
        clocks["window"] = ("about 1.2 s of replays of the same launches immediately before the "
                            "timed region, plus the timed region")

    # correctness spot check of the timed configuration (cheap): y vs a second
    # launch on another copy must be bit-identical (fixed reduction order)
    y_timed = y.clone()
    with torch.cuda.stream(stream):
        launch(1, stream)
    torch.cuda.synchronize(dev)
    deterministic = bool(torch.equal(y, y_timed))

    e2e = run_e2e(a, qw, copies, ncopies, x, M, N, K, sym, dev, stream, ws, ws_bytes, world)

    if not a.no_extras:
        extras["isolated"] = time_isolated(launch, stream, dev, algorithmic_bytes(M, N, K, sym))
        extras["read_ceiling"] = time_read_ceiling(dev, stream)
        extras["other_m"] = time_other_m(qw, copies, ncopies, N, K, sym, dev, stream)

    bytes_per = algorithmic_bytes(M, N, K, sym)
    us_per_launch = elapsed_ms * 1e3 / a.steps
    achieved_gbs = bytes_per / (us_per_launch * 1e-6) / 1e9
    peak, peak_src = measured_peaks()
    traffic = None
    if NCU_TRAFFIC["sources_sha256"] == kernel_sources_sha():
        traffic = NCU_TRAFFIC["bytes_per_launch"]
    value = elapsed_ms * 1e3 / (a.steps * world)

    line = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": elapsed_ms / a.steps,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "int32+f32",
        "data": "synthetic",
        "config": {"workload": "llama70b_down_8192x28672_asym_g128_m1", "N": N, "K": K, "M": M,
                   "group_size": 128, "symmetric": sym, "weights": "N(0,0.015) bf16, seeded PCG64",
                   "l2": f"rotating {ncopies} packed-weight copies "
                         f"({ncopies * wbytes / 1e6:.0f} MB > {l2 / 1e6:.0f} MB L2)",
                   "timing": "CUDA graphs of back-to-back GEMV launches, CUDA events; "
                             "host sync, then a ~0.25 ms device-side delay queued ahead "
                             "of the start event",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "us_per_linear_per_gpu": round(elapsed_ms * 1e3 / a.steps, 4),
        "hbm_tbs": round(achieved_gbs / 1e3, 4),
        "roofline": {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved_gbs / peak, 4), "traffic": traffic,
                     "bytes_per_launch": bytes_per, "peak_source": peak_src,
                     "frac_of_nominal_8tbs": round(achieved_gbs / 8000.0, 4)},
        "gpu_launches": 2 * a.steps,          # the streaming GEMV and its split-K finish per step
        "deterministic": deterministic,
        "e2e": e2e,
        "clocks": clocks,
    }
    if "read_ceiling" in extras:
        extras["read_ceiling"]["gemv_frac"] = round(achieved_gbs / extras["read_ceiling"]["gbs"], 4)
    if not a.no_extras:
        del copies, qw
        torch.cuda.empty_cache()
        extras["gemm"] = time_gemm(dev, stream)
        extras["layer_awq"] = time_layer_awq(dev, stream)
        extras["nvfp4"] = time_nvfp4(dev, stream)
        extras["gptq"] = time_gptq(dev, stream)
        extras["awq_search"] = time_awq_search(dev, stream)
    line.update(extras)
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(W, x, N, K, sym)
    return line


def soak_graph(launch, stream, chunk, dev):
    """One CUDA graph of `chunk` launches, replayed untimed to keep the GPU busy
    while the clock sampler watches."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(chunk):
            launch(i, stream)
    return g


def build_graphs(launch, stream, steps, chunk, dev):
    import torch
    graphs = []
    # make sure the first launch (one-time set-up) happens outside capture
    with torch.cuda.stream(stream):
        launch(0, stream)
    torch.cuda.synchronize(dev)
    sizes = [chunk] * (steps // chunk) + ([steps % chunk] if steps % chunk else [])
    cache = {}
    for n in sizes:
        if n not in cache:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    launch(i, stream)
            cache[n] = g
        graphs.append(cache[n])
    return graphs


def time_offline(Wt, qw, stream, N, K, sym):
    """Quantize + relayout timings for the same weight (events, 5 reps each;
    the 470 MB bf16 input exceeds L2)."""
    import torch
    from post_weight_quantization_wq_b200 import _binding as abi
    reps = 5
    d_status = torch.zeros(4, dtype=torch.int32, device=Wt.device)
    res = {}
    for name, fn in (
        ("quantize_rtn", lambda: abi.wq_quantize_rtn(Wt, None, N, K, 128, sym, qw.qweight,
                                                     qw.scales, qw.zeros, d_status, stream)),
        ("pack_layout", lambda: abi.wq_pack_layout(qw.qweight, qw.scales, qw.zeros, N, K, 128,
                                                   sym, 1, qw.packed, qw.packed.numel(),
                                                   stream))):
        fn()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            st = fn()
            assert st == 0
        e1.record(stream)
        e1.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / reps
        if name == "quantize_rtn":
            nbytes = 2 * N * K + N * K // 2 + 2 * N * K // 128 * (1 if sym else 2)
        else:
            nbytes = 2 * (N * K // 2 + 2 * N * K // 128 * (1 if sym else 2))
        res[name] = {"us": round(us, 2), "bytes": nbytes,
                     "gbs": round(nbytes / (us * 1e-6) / 1e9, 1)}
    return res


def time_isolated(launch, stream, dev, nbytes, reps=200, warm=20):
    """Single launches, each after an L2 flush (a 2x-L2 buffer is rewritten
    outside the timed pair of events): median, p10, p90 in microseconds."""
    import torch
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    ts = []
    with torch.cuda.stream(stream):
        for i in range(warm + reps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            launch(i, stream)
            e1.record(stream)
            e1.synchronize()
            if i >= warm:
                ts.append(e0.elapsed_time(e1) * 1e3)
    ts.sort()
    q = lambda f: ts[min(len(ts) - 1, int(f * len(ts)))]
    return {"us_median": round(q(0.5), 3), "us_p10": round(q(0.1), 3), "us_p90": round(q(0.9), 3),
            "gbs_median": round(nbytes / (q(0.5) * 1e-6) / 1e9, 1), "reps": reps,
            "protocol": "one launch per event pair after a 2xL2 flush, 20 warm-up"}


def time_read_ceiling(dev, stream, nbytes=2 << 30, reps=20):
    """Read-only HBM rate of this GPU: wq_stream_read_probe over a 2 GiB
    buffer (16-byte streaming loads), best and median of 20."""
    import torch
    from post_weight_quantization_wq_b200 import _binding as abi
    buf = torch.full((nbytes,), 7, dtype=torch.uint8, device=dev)
    out = torch.zeros(4, dtype=torch.int32, device=dev)
    ts = []
    with torch.cuda.stream(stream):
        for i in range(reps + 3):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            st = abi.wq_stream_read_probe(buf, nbytes, out, stream)
            e1.record(stream)
            e1.synchronize()
            assert st == 0
            if i >= 3:
                ts.append(e0.elapsed_time(e1) * 1e-3)
    ts.sort()
    del buf
    return {"gbs": round(nbytes / ts[0] / 1e9, 1), "gbs_median": round(nbytes / ts[len(ts) // 2] / 1e9, 1),
            "bytes": nbytes, "kernel": "wq_stream_read_probe (16-byte streaming loads, all SMs)"}


def time_gemm(dev, stream):
    """The tensor-core GEMM (wq_gemm_w4a16) at M = 16, 32, 64 on the two
    batched-decode shapes (28672x8192 and 8192x28672, asymmetric), graphs of
    back-to-back launches over copies of the packed weight (> L2)."""
    import numpy as np
    import torch
    import post_weight_quantization_wq_b200 as wq
    from post_weight_quantization_wq_b200 import _binding as abi
    from post_weight_quantization_wq_b200 import inputs
    out = {}
    cid = 4
    wl = inputs.WORKLOADS[cid]
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    for li, lin in enumerate(wl.linears):
        N, K = lin.N, lin.K
        W = inputs.workload_weight(cid, li)
        Wt = torch.from_numpy(W.view(np.int16)).to(dev).view(torch.bfloat16)
        del W
        qw = wq.quantize(Wt, symmetric=wl.sym, stream=stream)
        torch.cuda.synchronize(dev)
        del Wt
        ncopies = max(3, math.ceil(3 * l2 / qw.packed.numel()))
        copies = [qw.packed] + [qw.packed.clone() for _ in range(ncopies - 1)]
        bf16_peak = _measured_bf16_tflops()
        cases = [(M, 0) for M in wl.Ms] + [(M, 1) for M in wl.Ms]
        cases += [(M, 0) for M in ((128, 512, 2048) if li == 0 else (512,))]
        for M, forced in cases:
            ch = inputs.outlier_channels(K, 0.01, inputs.outlier_seed(cid, K))
            x = (inputs.workload_activations(cid, li, M) if M <= 64 else
                 inputs.activations(M, K, seed=M + li, channels=ch, mult=30.0))
            xt = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            ws_bytes = abi.wq_gemm_workspace_bytes(M, N, K)
            ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=dev)

            def launch(i, s):
                st = abi.wq_gemm_w4a16(xt, None, copies[i % ncopies], M, N, K, 128, wl.sym, 1, y,
                                       ws, ws_bytes, s)
                assert st == 0

            steps = 1000 if M <= 64 else (200 if M <= 512 else 40)
            abi.wq_debug_gemm_force_fold(forced)
            graphs = build_graphs(launch, stream, steps, min(50 * ncopies, steps), dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                for g in graphs[:2]:
                    g.replay()
                e0.record(stream)
                for g in graphs:
                    g.replay()
                e1.record(stream)
            e1.synchronize()
            abi.wq_debug_gemm_force_fold(0)
            us = e0.elapsed_time(e1) * 1e3 / steps
            b = algorithmic_bytes(M, N, K, wl.sym)
            tflops = 2.0 * M * N * K / (us * 1e-6) / 1e12
            rec = {"us": round(us, 3), "gbs": round(b / (us * 1e-6) / 1e9, 1),
                   "tflops": round(tflops, 1), "launches": steps + 1,
                   "kernel": ("many-row (fold)" if (forced or M > 64) else
                              "int8 decode" if (M <= 16 and K % 512 == 0) else "skinny")}
            if M > 64 and bf16_peak:
                rec["tensor_frac_of_measured_bf16"] = round(tflops / bf16_peak, 4)
            out[f"{N}x{K}_m{M}" + ("_fold" if forced else "")] = rec
        del copies, qw
        torch.cuda.empty_cache()
    if abi.wq_last_device_status(stream) != 0:
        raise RuntimeError("device error in the GEMM leg")
    return out


def time_layer_awq(dev, stream):
    """The AWQ workload: the seven linears of a Llama-70B GQA decoder layer
    (q, k, v, o, gate, up, down; 455 MB packed, more than L2) quantized with
    the AWQ scale folded in, run in order through wq_gemv_w4a16 with the
    activation factor 1/s, as one CUDA graph; M = 1 and 4.  Also each linear
    alone, over rotating copies of its weight (> 3 x L2)."""
    import numpy as np
    import torch
    import post_weight_quantization_wq_b200 as wq
    from post_weight_quantization_wq_b200 import _binding as abi
    from post_weight_quantization_wq_b200 import inputs
    cid = 5
    wl = inputs.WORKLOADS[cid]
    lins = []
    for li, lin in enumerate(wl.linears):
        W = inputs.workload_weight(cid, li)
        s_awq = inputs.workload_awq_scale(cid, li)
        Wt = torch.from_numpy(W.view(np.int16)).to(dev).view(torch.bfloat16)
        del W
        s_t = torch.from_numpy(s_awq).to(dev)
        qw = wq.quantize(Wt, awq_scale=s_t, symmetric=wl.sym, stream=stream)
        torch.cuda.synchronize(dev)
        del Wt
        inv = (1.0 / s_t.double()).float()
        lins.append((lin, qw, inv))
    out = {}
    for M in wl.Ms:
        runs = []
        nbytes = 0
        for li, (lin, qw, inv) in enumerate(lins):
            x = inputs.workload_activations(cid, li, M)
            xt = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
            y = torch.empty((M, lin.N), dtype=torch.float32, device=dev)
            wsb = abi.wq_workspace_bytes(M, lin.N, lin.K)
            ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device=dev)
            runs.append((lin, qw, inv, xt, y, ws, wsb))
            nbytes += algorithmic_bytes(M, lin.N, lin.K, wl.sym)

        def layer(s):
            for lin, qw, inv, xt, y, ws, wsb in runs:
                st = abi.wq_gemv_w4a16(xt, inv, qw.packed, M, lin.N, lin.K, 128, wl.sym, 1, y, ws,
                                       wsb, s)
                assert st == 0

        with torch.cuda.stream(stream):
            layer(stream)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        reps = 20
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                layer(stream)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            g.replay()
            e0.record(stream)
            for _ in range(10):
                g.replay()
            e1.record(stream)
        e1.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (10 * reps)
        # each linear alone: back-to-back launches over enough copies of its
        # packed weight to exceed L2 three times
        per = {}
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        for lin, qw, inv, xt, y, ws, wsb in runs:
            ncopies = max(3, math.ceil(3 * l2 / qw.packed.numel()))
            copies = [qw.packed] + [qw.packed.clone() for _ in range(ncopies - 1)]

            def one(i, s_):
                st = abi.wq_gemv_w4a16(xt, inv, copies[i % ncopies], M, lin.N, lin.K, 128, wl.sym,
                                       1, y, ws, wsb, s_)
                assert st == 0

            steps = 20 * ncopies
            gl = build_graphs(one, stream, steps, steps, dev)
            f0 = torch.cuda.Event(enable_timing=True)
            f1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                gl[0].replay()
                f0.record(stream)
                for _ in range(3):
                    gl[0].replay()
                f1.record(stream)
            f1.synchronize()
            per[lin.name] = round(f0.elapsed_time(f1) * 1e3 / (3 * steps), 2)
            del copies, gl
        out[f"m{M}"] = {"us_per_layer": round(us, 2), "bytes": nbytes,
                        "gbs": round(nbytes / (us * 1e-6) / 1e9, 1), "launches": 7,
                        "us_per_linear_alone": per}
    if abi.wq_last_device_status(stream) != 0:
        raise RuntimeError("device error in the AWQ layer leg")
    del lins
    torch.cuda.empty_cache()
    return out


# fp64 rate of a B200 from its unit counts: 148 SMs x 64 fp64 FMA per clock x
# 2 flops x 1.965 GHz (the calibrated quantizers run on fp64 CUDA cores).
FP64_PEAK_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12
# dense FP4 tensor rate: the measured bf16 GEMM rate x 4 (nominal FP4 / bf16)
FP4_PER_BF16 = 4.0


def _events_time(fn, stream, reps, warm=2):
    import torch
    with torch.cuda.stream(stream):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps          # ms


def time_nvfp4(dev, stream):
    """NVFP4 (W4A4, block-scaled FP4 tensor cores, wq_nvfp4_linear): the
    8192x28672 down projection at M = 1 and 16 (decode, HBM-bound: 4.5 bits
    per weight) and the 28672x8192 gate/up projection at M = 128 (a batch of
    activation rows, reported against the FP4 tensor rate); graphs of
    back-to-back calls over copies of the packed weight (> L2)."""
    import numpy as np
    import torch
    import post_weight_quantization_wq_b200 as wq
    from post_weight_quantization_wq_b200 import _binding as abi
    from post_weight_quantization_wq_b200 import inputs
    out = {}
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    bf16_peak = _measured_bf16_tflops()
    for (cid, li), Ms in (((3, 3), (1, 16)), ((4, 0), (128,))):
        W = inputs.workload_weight(cid, li)
        N, K = W.shape
        Wt = torch.from_numpy(W.view(np.int16)).to(dev).view(torch.bfloat16)
        del W
        with torch.cuda.stream(stream):
            qw = wq.nvfp4_quantize(Wt, stream=stream)
        torch.cuda.synchronize(dev)
        del Wt
        ncopies = max(3, math.ceil(3 * l2 / qw.packed.numel()))
        copies = [qw.packed] + [qw.packed.clone() for _ in range(ncopies - 1)]
        for M in Ms:
            x = inputs.activations(M, K, seed=M + 11)
            xt = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            wsb = abi.wq_nvfp4_linear_workspace_bytes(M, N, K)
            ws = torch.empty(wsb, dtype=torch.uint8, device=dev)

            def launch(i, s):
                st = abi.wq_nvfp4_linear(xt, copies[i % ncopies], qw.tensor_scale, M, N, K, y, ws,
                                         wsb, s)
                assert st == 0

            steps = 400
            graphs = build_graphs(launch, stream, steps, 20 * ncopies, dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                graphs[0].replay()
                e0.record(stream)
                for g in graphs:
                    g.replay()
                e1.record(stream)
            e1.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / steps
            nbytes = N * K // 2 + N * K // 16 + 2 * M * K + 4 * M * N
            tflops = 2.0 * M * N * K / (us * 1e-6) / 1e12
            rec = {"us": round(us, 3), "gbs": round(nbytes / (us * 1e-6) / 1e9, 1),
                   "tflops": round(tflops, 1), "bytes": nbytes}
            if M >= 128 and bf16_peak:
                rec["fp4_tensor_frac"] = round(tflops / (bf16_peak * FP4_PER_BF16), 4)
            out[f"{N}x{K}_m{M}"] = rec
        del copies, qw
        torch.cuda.empty_cache()
    if abi.wq_last_device_status(stream) != 0:
        raise RuntimeError("device error in the NVFP4 leg")
    return out


def _measured_bf16_tflops():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return None


def time_gptq(dev, stream, N=4096, K=4096, T=512):
    """GPTQ on a 4096 x 4096 weight (a Llama-7B attention projection) with 512
    correlated calibration rows (wq_gptq_quantize: fp64 Hessian, Cholesky,
    per-group feedback); fp64 flops counted from the algorithm's steps."""
    import numpy as np
    import torch
    import post_weight_quantization_wq_b200 as wq
    from post_weight_quantization_wq_b200 import _binding as abi
    from post_weight_quantization_wq_b200 import inputs
    W = torch.from_numpy(inputs.weights(N, K, 0.02, seed=31).view(np.int16)).to(dev).view(torch.bfloat16)
    X = torch.from_numpy(inputs.correlated_calibration(T, K, seed=32).view(np.int16)).to(dev).view(
        torch.bfloat16)
    ws = torch.empty(abi.wq_gptq_workspace_bytes(T, N, K), dtype=torch.uint8, device=dev)
    ms = _events_time(lambda: wq.gptq_quantize(W, X, workspace=ws, stream=stream), stream, 3, 1)
    flops = 2.0 * T * K * K + K ** 3 / 3.0 + 2.0 * N * K * K / 2 + (K // 128) * 2.0 * N * 128 * 128
    return {"shape": f"{N}x{K}", "calib_rows": T, "ms": round(ms, 2),
            "fp64_tflops": round(flops / (ms * 1e-3) / 1e12, 2),
            "fp64_peak_tflops_derived": round(FP64_PEAK_TFLOPS, 1)}


def time_awq_search(dev, stream):
    """The AWQ alpha search (21 values) on the decoder layer's q projection
    (8192 x 8192) with its 128 calibration rows; the loss of each alpha is an
    fp64 product of the calibration rows with the weight difference."""
    import numpy as np
    import torch
    import post_weight_quantization_wq_b200 as wq
    from post_weight_quantization_wq_b200 import _binding as abi
    from post_weight_quantization_wq_b200 import inputs
    cid, li = 5, 0
    wl = inputs.WORKLOADS[cid]
    K = wl.linears[li].K
    W = inputs.workload_weight(cid, li)
    N = W.shape[0]
    X = inputs.activations(wl.calib_rows, K, inputs.calib_seed(cid, K),
                           inputs.outlier_channels(K, wl.act_outlier_frac, inputs.outlier_seed(cid, K)),
                           wl.calib_outlier_mult)
    Wt = torch.from_numpy(W.view(np.int16)).to(dev).view(torch.bfloat16)
    Xt = torch.from_numpy(X.view(np.int16)).to(dev).view(torch.bfloat16)
    T = X.shape[0]
    ws = torch.empty(abi.wq_awq_search_workspace_bytes(T, N, K, 20), dtype=torch.uint8, device=dev)
    res = {}

    def run():
        res.update(wq.awq_search(Wt, Xt, workspace=ws, stream=stream))
    ms = _events_time(run, stream, 2, 1)
    flops = 21 * 2.0 * T * N * K
    return {"shape": f"{N}x{K}", "calib_rows": T, "grid": 21, "ms": round(ms, 2),
            "alpha": res.get("alpha"), "fp64_tflops": round(flops / (ms * 1e-3) / 1e12, 2),
            "fp64_peak_tflops_derived": round(FP64_PEAK_TFLOPS, 1)}


def time_other_m(qw, copies, ncopies, N, K, sym, dev, stream):
    """The same weight at M = 2, 4, 8 through the CUDA-core GEMV, and at
    M = 4, 8 through the tensor-core GEMM (2000 launches each, graphs)."""
    import numpy as np
    import torch
    from post_weight_quantization_wq_b200 import _binding as abi
    from post_weight_quantization_wq_b200 import inputs
    out = {}
    for path, Ms in (("gemv", (2, 4, 8)), ("gemm", (4, 8))):
        fn = abi.wq_gemv_w4a16 if path == "gemv" else abi.wq_gemm_w4a16
        for M in Ms:
            x = inputs.workload_activations(WORKLOAD_CID, WORKLOAD_LIN, M)
            xt = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            ws_bytes = (abi.wq_workspace_bytes if path == "gemv" else abi.wq_gemm_workspace_bytes)(M, N, K)
            ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=dev)

            def launch(i, s):
                st = fn(xt, None, copies[i % ncopies], M, N, K, 128, sym, 1, y, ws, ws_bytes, s)
                assert st == 0

            steps = 2000
            graphs = build_graphs(launch, stream, steps, 100 * ncopies, dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                for g in graphs[:2]:
                    g.replay()
                e0.record(stream)
                for g in graphs:
                    g.replay()
                e1.record(stream)
            e1.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / steps
            b = algorithmic_bytes(M, N, K, sym)
            key = str(M) if path == "gemv" else f"{M}_tensor_cores"
            out[key] = {"us": round(us, 3), "gbs": round(b / (us * 1e-6) / 1e9, 1), "entry": fn.__name__}
    return out


def run_e2e(a, qw, copies, ncopies, x, M, N, K, sym, dev, stream, ws, ws_bytes, world):
    """Each step: pinned host x -> device, GEMV through the public binding,
    device y -> pinned host; timed with events around all steps."""
    import numpy as np
    import torch
    from post_weight_quantization_wq_b200 import _binding as abi
    steps = min(a.steps, 20000)
    x_host = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((M, N), dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(x_host, device=dev)
    y_dev = torch.empty((M, N), dtype=torch.float32, device=dev)
    with torch.cuda.stream(stream):
        for i in range(min(a.warmup, 50)):
            x_dev.copy_(x_host, non_blocking=True)
            abi.wq_gemv_w4a16(x_dev, None, copies[i % ncopies], M, N, K, 128, sym, 1, y_dev,
                              ws, ws_bytes, stream)
            y_host.copy_(y_dev, non_blocking=True)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(steps):
            x_dev.copy_(x_host, non_blocking=True)
            st = abi.wq_gemv_w4a16(x_dev, None, copies[i % ncopies], M, N, K, 128, sym, 1,
                                   y_dev, ws, ws_bytes, stream)
            if st != 0:
                raise RuntimeError(abi.status_string(st))
            y_host.copy_(y_dev, non_blocking=True)
        e1.record(stream)
    e1.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    barrier(world)
    return {"value": round(ms * 1e3 / (steps * world), 4), "unit": UNIT,
            "h2d_bytes_per_step": x_host.numel() * 2, "d2h_bytes_per_step": y_host.numel() * 4,
            "steps": steps, "path": "pinned host x -> device, wq_gemv_w4a16 via ctypes, "
                                    "device y -> pinned host, per step from Python"}


def cpu_baseline(W, x, N, K, sym, target_s: float = 10.0):
    """The CPU oracle (plain C, fp64) on a bounded sample of output rows of the
    same linear, scaled to one full linear: once single-threaded, once on all
    host cores (the unchanged oracle called on disjoint row ranges from one
    thread per core; the C call releases the GIL)."""
    import concurrent.futures as cf
    import numpy as np
    import oracle
    rows0 = 64
    q, s, z, _ = oracle.quantize_bf16(W[:rows0], None, sym=sym)
    P = oracle.pack_u4(q, sym)
    t = time.perf_counter()
    oracle.linear(x, P, s, z, K, sym=sym)
    per_row = (time.perf_counter() - t) / rows0
    R = int(min(N, max(rows0, target_s / max(per_row, 1e-9))))
    tq = time.perf_counter()
    q, s, z, _ = oracle.quantize_bf16(W[:R], None, sym=sym)
    quant_single = (time.perf_counter() - tq) / R * N * 1e6
    P = oracle.pack_u4(q, sym)
    del q
    t = time.perf_counter()
    oracle.linear(x, P, s, z, K, sym=sym)
    el = time.perf_counter() - t
    single = el / R * N * 1e6
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    chunks = [np.arange(i, min(R, i + max(1, R // cores)), dtype=np.int64)
              for i in range(0, R, max(1, R // cores))]
    t = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=cores) as ex:
        list(ex.map(lambda r: oracle.linear(x, P, s, z, K, sym=sym, rows=r), chunks))
    el_mt = time.perf_counter() - t
    multi = el_mt / R * N * 1e6
    return {"value": round(multi, 1), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{R} of {N} output rows of the 8192x28672 linear at M=1 (fp64 C oracle, "
                      f"dequantize + dot per row) on {cores} threads ({el_mt:.2f} s) and on one "
                      f"thread ({el:.1f} s), scaled to the full linear",
            "single_thread_value": round(single, 1),
            "quantize_single_thread_us": round(quant_single, 1),
            "host_cpu": _cpu_model(), "host_cores_available": os.cpu_count()}


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return None


# ------------------------------------------------------------------ reference arm

def run_reference(a, rank: int, world: int):
    """The CPU oracle as the reference arm: each step computes one output row
    of the 8192 x 28672 linear at M = 1 (dequantize + fp64 dot), cycling over
    the rows of a sampled block; value = mean step time x N."""
    import numpy as np
    import oracle
    from post_weight_quantization_wq_b200 import inputs
    wl = inputs.WORKLOADS[WORKLOAD_CID]
    lin = wl.linears[WORKLOAD_LIN]
    N, K, sym = lin.N, lin.K, wl.sym
    W = inputs.workload_weight(WORKLOAD_CID, WORKLOAD_LIN)
    x = inputs.workload_activations(WORKLOAD_CID, WORKLOAD_LIN, 1)
    R = 256
    q, s, z, _ = oracle.quantize_bf16(W[:R], None, sym=sym)
    P = oracle.pack_u4(q, sym)
    del W, q
    rows = [np.array([i], np.int64) for i in range(R)]
    for i in range(a.warmup):
        oracle.linear(x, P, s, z, K, sym=sym, rows=rows[i % R])
    # bound the run: at most ~60 s of steps
    t0 = time.perf_counter()
    oracle.linear(x, P, s, z, K, sym=sym, rows=rows[0])
    per = time.perf_counter() - t0
    steps = min(a.steps, max(1, int(60.0 / max(per, 1e-9))))
    t0 = time.perf_counter()
    for i in range(steps):
        oracle.linear(x, P, s, z, K, sym=sym, rows=rows[i % R])
    el = time.perf_counter() - t0
    value = el / steps * N * 1e6
    sample = (f"{steps} steps of one output row each (rows 0..{R - 1} of the 8192x28672 linear, "
              f"M=1, fp64 C oracle), mean step time x {N} rows")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT,
        "n_gpus": world, "steps": steps, "warmup": a.warmup, "ms_per_step": el / steps * 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "llama70b_down_8192x28672_asym_g128_m1", "N": N, "K": K, "M": 1,
                   "group_size": 128, "symmetric": sym},
        "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ------------------------------------------------------------------ distributed

def barrier(world):
    if world > 1:
        import torch.distributed as tdist
        tdist.barrier()


def max_over_ranks(v, world, dev):
    if world == 1:
        return v
    import torch
    import torch.distributed as tdist
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def run_case(a):
    """A few launches of one kernel on one workload, for profilers: gemv_m1 /
    gemv_m4 = wq_gemv_w4a16 on 8192x28672 at M = 1 (CUDA cores) / 4 (int8
    tensor cores); gemm_m16 / gemm_m64 / gemm_m512 = wq_gemm_w4a16 on
    28672x8192 at M = 16 (int8 tensor cores) / 64 (bf16 skinny kernel) / 512
    (many-row prefill kernel), asymmetric; nvfp4_m1 / nvfp4_m128 =
    wq_nvfp4_linear on 8192x28672 at M = 1 / 28672x8192 at M = 128.  About
    1 GB on the device."""
    import numpy as np
    import torch
    import post_weight_quantization_wq_b200 as wq
    from post_weight_quantization_wq_b200 import inputs
    if a.case.startswith("nvfp4"):
        cid, li, M = {"nvfp4_m1": (WORKLOAD_CID, WORKLOAD_LIN, 1), "nvfp4_m128": (4, 0, 128)}[a.case]
        W = inputs.workload_weight(cid, li)
        Wt = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
        x = inputs.activations(M, W.shape[1], seed=M + 11)
        del W
        qw = wq.nvfp4_quantize(Wt)
        del Wt
        xt = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
        for _ in range(3):
            y = wq.nvfp4_linear(xt, qw)
        torch.cuda.synchronize()
        if wq.last_device_status() != 0:
            raise RuntimeError("device error")
        print(json.dumps({"case": a.case, "y_sum": float(y.double().sum())}))
        return
    cid, li, M = {"gemv_m1": (WORKLOAD_CID, WORKLOAD_LIN, 1),
                  "gemv_m4": (WORKLOAD_CID, WORKLOAD_LIN, 4), "gemm_m16": (4, 0, 16),
                  "gemm_m64": (4, 0, 64), "gemm_m512": (4, 0, 512)}[a.case]
    W = inputs.workload_weight(cid, li)
    x = (inputs.workload_activations(cid, li, M) if M in inputs.WORKLOADS[cid].Ms else
         inputs.activations(M, W.shape[1], seed=M + 11))
    Wt = torch.from_numpy(W.view(np.int16)).cuda().view(torch.bfloat16)
    del W
    qw = wq.quantize(Wt, symmetric=inputs.WORKLOADS[cid].sym)
    del Wt
    xt = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    path = "gemm" if a.case.startswith("gemm") else "gemv"
    for _ in range(3):
        y = wq.linear(xt, qw, path=path)
    torch.cuda.synchronize()
    if wq.last_device_status() != 0:
        raise RuntimeError("device error")
    print(json.dumps({"case": a.case, "y_sum": float(y.double().sum())}))


def main():
    a = _args()
    if a.case:
        run_case(a)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(a, rank, world)), flush=True)
        return
    if world > 1:
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=dt.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(a, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as tdist
            tdist.destroy_process_group()


if __name__ == "__main__":
    main()
