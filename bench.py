"""Benchmark of the block-wise FP8 linear layer hot path on B200.

One step = one pass of the whole hot path over one Llama-3.1-8B-shaped layer
at M = 8192 prefill tokens (4 x 2048), FP32 block scales:
  - per-step recalibration of the layer's four weight tensors
    (QKV 6144x4096, O 4096x4096, gate+up 28672x4096, down 4096x14336) into
    E4M3 codes + 128x128 scales, one launch;
  - for each of the four linears: 1x128 quantization of its bf16 input and the
    block-scaled FP8 GEMM (FP32 promotion, bf16 out).
Metric: FP8 GEMM throughput of the step in TFLOP/s (GEMM FLOPs of the four
linears / step time, so the quantization and recalibration time counts
against it).  Per-row figures (quantize / recalibrate GB/s, each GEMM's
TFLOP/s) are reported under "rows".

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun (N > 1) every rank runs the same single-GPU workload on its own
GPU (replicas: the path has no exchange step); value = all ranks' FLOPs / the
slowest rank's time.

--impl reference times the CPU oracle (oracle/) on the host cores on a bounded
sample of the same workload (the slow reference program; parity and the
roofline fraction are the headline, not this ratio).
"""
import argparse
import hashlib
import itertools
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import fp8bq_workloads as wl  # noqa: E402

METRIC = "block-scaled FP8 GEMM TFLOP/s (% of dense FP8 peak); quantize/recal GB/s (% HBM)"
WORKLOAD = "llama3.1-8b-shaped prefill layer: 4 linears (qkv, o, gate_up, down) at M=8192 tokens, fp32 block scales"
NAMES = list(wl.LLAMA8B_SHAPES)
M_TOKENS = wl.PREFILL_TOKENS
LAUNCHES_PER_STEP = 1 + 2 * len(NAMES)        # recalibrate + (quant_act + gemm) per linear


def gemm_flops_step():
    return sum(2.0 * M_TOKENS * N * K for N, K in wl.LLAMA8B_SHAPES.values())


def quant_act_bytes(M, K):
    """bf16 in + E4M3 out + one fp32 scale per 128 elements."""
    return M * K * 2 + M * K + M * ((K + 127) // 128) * 4


def recal_bytes(N, K):
    return N * K * 2 + N * K + ((N + 127) // 128) * ((K + 127) // 128) * 4


def gemm_bytes(M, N, K):
    return M * K + N * K + M * N * 2 + M * (K // 128) * 4 + ((N + 127) // 128) * (K // 128) * 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _strip_comments(src):
    """C/C++ source without its comments and with every run of whitespace
    outside string and character literals folded to one space, so that an
    edit of comments or layout leaves the fingerprint of the code unchanged."""
    out, i, n = [], 0, len(src)

    def space():
        if out and out[-1] != " ":
            out.append(" ")
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
            space()
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            space()
        elif c.isspace():
            space()
            i += 1
        else:
            out.append(c)
            i += 1
    return "".join(out).strip()


def kernel_source_sha():
    """Fingerprint of the GEMM kernel's code (its sources without comments)."""
    h = hashlib.sha256()
    for f in ("gemm.cu", "gemm_promote.cuh", "device.cuh", "quant.cuh", "raster.cu"):
        src = open(os.path.join(ROOT, "fp8_block_scaled_fp8bq_b200", "csrc", f), encoding="utf-8").read()
        h.update(_strip_comments(src).encode("utf-8"))
    return h.hexdigest()[:16]


def committed_traffic():
    """DRAM bytes per GEMM launch from the committed ncu summary, if the kernel is unchanged.

    The summary holds `key: value` lines; `source_sha` names the kernel sources
    the counters were taken from and `dram_bytes_per_launch_step_avg` is the
    mean over the step's four GEMM launches of dram__bytes_read.sum +
    dram__bytes_write.sum."""
    p = os.path.join(ROOT, "profiles", "gemm_traffic_llama8b_layer_M8192.txt")
    if not os.path.exists(p):
        return None
    d = {}
    for line in open(p):
        if ":" in line and not line.startswith((" ", "#", "`")):
            k, v = line.split(":", 1)
            d[k.strip()] = v.strip()
    if d.get("source_sha") != kernel_source_sha():
        return None
    try:
        return int(d["dram_bytes_per_launch_step_avg"])
    except (KeyError, ValueError):
        return None


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clocks_setting"}

    def __init__(self, device_index, period_s=0.02):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                self.reasons |= self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if self.nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# --------------------------------------------------------------------------- our arm
class LayerStep:
    """Device buffers and the launch sequence of one step."""

    def __init__(self, fq, device, seed=0, mode=0):
        self.fq = fq
        self.mode = mode
        self.x, self.w, self.q_w, self.s_w, self.q_a, self.s_a, self.y = {}, {}, {}, {}, {}, {}, {}
        layer = wl.llama_layer(seed=seed, M=M_TOKENS, device=device)
        for name, (N, K) in wl.LLAMA8B_SHAPES.items():
            x, w = layer[name]
            self.x[name], self.w[name] = x, w
            self.q_w[name] = torch.empty((N, K), dtype=torch.uint8, device=device)
            self.s_w[name] = torch.empty((fq.ceil_div(N, 128), fq.ceil_div(K, 128)), dtype=torch.float32,
                                         device=device)
            self.q_a[name] = torch.empty((M_TOKENS, K), dtype=torch.uint8, device=device)
            self.s_a[name] = torch.empty(fq.act_scale_shape(M_TOKENS, K), dtype=torch.float32, device=device)
            self.y[name] = torch.empty((M_TOKENS, N), dtype=torch.bfloat16, device=device)
        self.recal_list = [(self.w[n], self.q_w[n], self.s_w[n]) for n in NAMES]

    def run(self, events=None, io=None):
        """One step.  events: optional dict name -> list of (start, end) CUDA events to record.
        io: optional (x, w, y) dicts of device buffers to use instead of the step's own
        inputs and outputs (the end-to-end run alternates two such sets)."""
        fq = self.fq
        x, w, y = io if io is not None else (self.x, self.w, self.y)
        recal_list = self.recal_list if io is None else [(w[n], self.q_w[n], self.s_w[n]) for n in NAMES]

        def ev(key):
            if events is None:
                return None
            e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            events.setdefault(key, []).append(e)
            return e

        e = ev("recalibrate")
        if e:
            e[0].record()
        fq.recalibrate(recal_list, self.mode)
        if e:
            e[1].record()
        for name in NAMES:
            e = ev("quant_act:" + name)
            if e:
                e[0].record()
            fq.quant_act(x[name], self.mode, q=self.q_a[name], sa=self.s_a[name])
            if e:
                e[1].record()
            e = ev("gemm:" + name)
            if e:
                e[0].record()
            fq.gemm(self.q_a[name], self.s_a[name], self.q_w[name], self.s_w[name], self.mode, out=y[name])
            if e:
                e[1].record()


def timed_steps(step, K, W, rank_sync):
    """Run W warm-up steps, then K timed steps; returns (seconds, events)."""
    for _ in range(W):
        step.run()
    torch.cuda.synchronize()
    rank_sync()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    events = {}
    start.record()
    for _ in range(K):
        step.run(events)
    end.record()
    torch.cuda.synchronize()
    rank_sync()
    torch.cuda.synchronize()
    return start.elapsed_time(end) / 1e3, events


def e2e_steps(fq, step, K, rank_sync):
    """The same step through the public API with host buffers: every step copies
    its inputs (activations and bf16 weights) from pinned host memory and its
    outputs back.  Steps are pipelined over two sets of device inputs/outputs and
    three streams, so the host-to-device copies of step k+1 run while step k
    computes and its outputs travel back (PCIe is full duplex); every step still
    moves all of its own bytes inside the timed region."""
    host_x = {n: step.x[n].cpu().pin_memory() for n in NAMES}
    host_w = {n: step.w[n].cpu().pin_memory() for n in NAMES}
    host_y = {n: torch.empty(step.y[n].shape, dtype=torch.bfloat16).pin_memory() for n in NAMES}
    h2d = sum(t.numel() * t.element_size() for t in list(host_x.values()) + list(host_w.values()))
    d2h = sum(t.numel() * t.element_size() for t in host_y.values())
    io = [(step.x, step.w, step.y),
          ({n: torch.empty_like(step.x[n]) for n in NAMES}, {n: torch.empty_like(step.w[n]) for n in NAMES},
           {n: torch.empty_like(step.y[n]) for n in NAMES})]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    s_comp = torch.cuda.current_stream()
    comp_done = [None, None]
    out_done = [None, None]

    def one(k):
        slot = k & 1
        x, w, y = io[slot]
        with torch.cuda.stream(s_in):
            if comp_done[slot] is not None:
                s_in.wait_event(comp_done[slot])        # step k-2 has finished reading this slot
            for n in NAMES:
                x[n].copy_(host_x[n], non_blocking=True)
                w[n].copy_(host_w[n], non_blocking=True)
            in_done = torch.cuda.Event()
            in_done.record(s_in)
        s_comp.wait_event(in_done)
        if out_done[slot] is not None:
            s_comp.wait_event(out_done[slot])           # step k-2's outputs have left this slot
        step.run(io=io[slot])
        comp_done[slot] = torch.cuda.Event()
        comp_done[slot].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[slot])
            for n in NAMES:
                host_y[n].copy_(y[n], non_blocking=True)
            out_done[slot] = torch.cuda.Event()
            out_done[slot].record(s_out)

    one(0)
    one(1)
    torch.cuda.synchronize()
    rank_sync()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_comp)
    s_in.wait_stream(s_comp)
    s_out.wait_stream(s_comp)
    for k in range(K):
        one(k)
    s_comp.wait_stream(s_out)
    s_comp.wait_stream(s_in)
    t1.record(s_comp)
    torch.cuda.synchronize()
    rank_sync()
    return t0.elapsed_time(t1) / 1e3, h2d, d2h


def cpu_baseline_oracle(budget_s=15.0):
    """The oracle on a bounded sample of the step, on the host cores.

    Sample: quantization of R rows of each linear's input, the oracle GEMM of
    those rows against the full weight, and the 128x128 quantization of the
    full weight; the time of a full step is extrapolated (rows scale
    linearly) and the metric is GEMM FLOPs / extrapolated step time.
    """
    import oracle
    R = max(1, oracle.num_threads())
    t_weight = 0.0
    t_rows = 0.0
    for i, (name, (N, K)) in enumerate(wl.LLAMA8B_SHAPES.items()):
        x = wl.activations(R, K, seed=100 + i)
        w = wl.weights(N, K, seed=200 + i)
        xb = x.view(torch.int16).numpy().view(np.uint16)
        wb = w.view(torch.int16).numpy().view(np.uint16)
        t0 = time.perf_counter()
        qw, sw = oracle.quant_weight(wb, 0)
        t1 = time.perf_counter()
        qa, sa = oracle.quant_act(xb, 0)
        oracle.gemm(qa, sa, qw, sw)
        t2 = time.perf_counter()
        t_weight += t1 - t0
        t_rows += t2 - t1
    step_s = t_weight + t_rows * (M_TOKENS / R)
    return {"value": gemm_flops_step() / step_s / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "%d rows of each of the 4 linears (act quant + FP64 GEMM) plus the full 128x128 weight "
                      "quantization; step time extrapolated to M=%d rows" % (R, M_TOKENS),
            "sample_seconds": round(t_weight + t_rows, 2)}


L2_BYTES = 126 * 2 ** 20


def rotations(nbytes):
    """Copies of a call's inputs to cycle through so that no call finds its
    operands in L2 left there by the previous one (at least 4x L2 in total)."""
    return max(1, -(-4 * L2_BYTES // max(1, nbytes)))


def graph_ms(calls, reps=3):
    """Per-call device time of `calls` (a list of no-argument launch functions),
    replayed as one CUDA graph so the host does not pace the GPU; the median
    of `reps` replays after one warm replay."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for fn in calls:
            fn()
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        g.replay()
        t1.record()
        torch.cuda.synchronize()
        times.append(t0.elapsed_time(t1) / len(calls))
    del g
    return statistics.median(times)


def oracle_row(work, secs, unit_scale, unit, sample, extrapolated_from=None):
    """The oracle's rate on a bounded sample, in the row's own unit."""
    import oracle
    d = {"value": work / secs / unit_scale, "unit": unit, "cores": oracle.num_threads(), "kind": "oracle",
         "sample": sample, "sample_seconds": round(secs if extrapolated_from is None else extrapolated_from, 3)}
    return d


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def config_rows(fq, dev, peaks, gemm_ms_step):
    """Every configuration of the workload besides the step itself: the single
    linear, the whole-model power-of-2 recalibration, the 16 decode-shaped
    linears (whole call, quantization included) and the two MoE expert GEMMs;
    each timed on the device and, beside it, the oracle on a bounded sample of
    the same work on the host cores.  Also the recalibration-overhead proxy."""
    import oracle
    rows = {}
    hbm = peaks["hbm_gbs"]
    fp8 = 2.0 * peaks["bf16_tflops"]

    # --- single block-scaled linear: quantize X and W, FP8 GEMM (3 launches)
    x, w = wl.single_linear(seed=0)
    M, K = x.shape
    N = w.shape[0]
    n = rotations(M * K * 2 + N * K * 2)
    xs = [x.to(dev) for _ in range(n)]
    ws_ = [w.to(dev) for _ in range(n)]
    qa = torch.empty((M, K), dtype=torch.uint8, device=dev)
    sa = torch.empty(fq.act_scale_shape(M, K), dtype=torch.float32, device=dev)
    qw = torch.empty((N, K), dtype=torch.uint8, device=dev)
    sw = torch.empty((N // 128, K // 128), dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

    def lin(i):
        def f():
            fq.quant_act(xs[i], fq.SCALE_FP32, q=qa, sa=sa)
            fq.quant_weight(ws_[i], fq.SCALE_FP32, q=qw, sw=sw)
            fq.gemm(qa, sa, qw, sw, fq.SCALE_FP32, out=y)
        return f
    ms = graph_ms([lin(i) for i in range(n)])
    fl = 2.0 * M * N * K
    t0 = time.perf_counter()
    oqa, osa = oracle.quant_act(bits(x), 0)
    oqw, osw = oracle.quant_weight(bits(w), 0)
    oracle.gemm(oqa, osa, oqw, osw)
    ot = time.perf_counter() - t0
    rows["single_linear:256x512x512"] = {
        "us_per_call": round(ms * 1e3, 2), "tflops": round(fl / (ms / 1e3) / 1e12, 3), "launches": 3,
        "note": "latency-bound (0.13 GFLOP); quant_act + quant_weight + gemm in a CUDA graph",
        "cpu_oracle": oracle_row(fl, ot, 1e12, "TFLOP/s", "the whole single linear")}
    del xs, ws_

    # --- decode-shaped linears: weights pre-quantized 128x128, X quantized inside the call
    for name, (N, K) in wl.LLAMA8B_SHAPES.items():
        wbf = wl.weights(N, K, seed=2)
        wq, wsc = fq.quant_weight(wbf.to(dev), fq.SCALE_FP32)
        oqw, osw = oracle.quant_weight(bits(wbf), 0)     # the oracle's own pre-quantized weight
        # oracle: one row (act quant + FP64 GEMM against the whole weight); the
        # time of M rows is M times that (rows are independent)
        xb = bits(wl.activations(1, K, seed=1))
        t0 = time.perf_counter()
        oqa, osa = oracle.quant_act(xb, 0)
        oracle.gemm(oqa, osa, oqw, osw)
        t_row = time.perf_counter() - t0
        for M in wl.DECODE_TOKENS:
            nbytes = decode_bytes(M, N, K)
            n = rotations(N * K)
            qws = [wq] + [wq.clone() for _ in range(n - 1)]
            x = wl.activations(M, K, seed=1, device=dev)
            out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            wsp = torch.zeros(max(256, fq.gemm_decode_workspace_size(M, N, K)), dtype=torch.uint8, device=dev)
            calls = [(lambda q=q: fq.gemm_decode(x, q, wsc, fq.SCALE_FP32, out=out, ws=wsp)) for q in qws]
            ms = graph_ms(calls * max(1, 64 // n))
            gbs = nbytes / (ms / 1e3) / 1e9
            ot = t_row * M
            rows["decode:%s:M%d" % (name, M)] = {
                "us_per_call": round(ms * 1e3, 2), "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                "bytes": nbytes, "tflops": round(2.0 * M * N * K / (ms / 1e3) / 1e12, 1),
                "cpu_oracle": oracle_row(nbytes, ot, 1e9, "GB/s",
                                         "one row (act quant + FP64 GEMM against the whole weight), "
                                         "time scaled to %d rows" % M)}
            del qws
        del wq, wsc, oqw, osw

    # --- the prefill GEMMs with power-of-2 scales (the native block-scaled
    # MMA, what fp8bq_gemm runs for them), M = 8192, inputs quantized once
    for name, (N, K) in wl.LLAMA8B_SHAPES.items():
        xa = wl.activations(M_TOKENS, K, seed=3, device=dev)
        wq_ = wl.weights(N, K, seed=4, device=dev)
        qa2, sa2 = fq.quant_act(xa, fq.SCALE_POW2)
        qw2, sw2 = fq.quant_weight(wq_, fq.SCALE_POW2)
        del xa, wq_
        y2 = torch.empty((M_TOKENS, N), dtype=torch.bfloat16, device=dev)
        # operand copies cycled so that no call finds its inputs in L2
        nr = rotations(M_TOKENS * K + N * K)
        ops = [(qa2, qw2)] + [(qa2.clone(), qw2.clone()) for _ in range(nr - 1)]
        ms = graph_ms([(lambda a=a, b=b: fq.gemm(a, sa2, b, sw2, fq.SCALE_POW2, out=y2)) for a, b in ops] *
                      max(1, 8 // nr))
        tf = 2.0 * M_TOKENS * N * K / (ms / 1e3) / 1e12
        rows["gemm_pow2:" + name] = {"ms": round(ms, 4), "tflops": round(tf, 1), "frac_fp8_peak": round(tf / fp8, 3),
                                     "kernel": "gemm_native_kernel (block-scaled MMA, UE8M0 scale factors)"}
        del qa2, sa2, qw2, sw2, y2, ops

    # --- MoE expert GEMMs (Qwen3-30B-A3B-shaped, Zipf top-8 routing)
    moe = wl.moe_layer(seed=0, device=dev)
    off = moe["offsets"].to(torch.int32).to(dev)
    offs = moe["offsets"].numpy()
    for what in ("up", "down"):
        x, w = moe["x_" + what], moe["w_" + what]
        E, N, K = w.shape
        R = x.shape[0]
        qa, sa = fq.quant_act(x, fq.SCALE_FP32)
        qw, sw = fq.quant_weight(w.reshape(E * N, K), fq.SCALE_FP32)
        qw, sw = qw.view(E, N, K), sw.view(E, N // 128, K // 128)
        y = torch.empty((R, N), dtype=torch.bfloat16, device=dev)
        ms = graph_ms([lambda: fq.grouped_gemm(qa, sa, qw, sw, off, fq.SCALE_FP32, out=y)] * 10)
        nbytes = moe_bytes(R, E, N, K)
        fl = 2.0 * R * N * K
        gbs = nbytes / (ms / 1e3) / 1e9
        sample = np.unique(np.concatenate([np.arange(offs[e], min(offs[e + 1], offs[e] + 1)) for e in range(E)]))
        oqa, osa = oracle.quant_act(bits(x), 0)
        oqw, osw = oracle.quant_weight(bits(w.reshape(E * N, K)), 0)
        oqw, osw = oqw.reshape(E, N, K), osw.reshape(E, N // 128, K // 128)
        t0 = time.perf_counter()
        oracle.grouped_gemm(oqa, osa, oqw, osw, offs, rows=sample)
        ot = (time.perf_counter() - t0) * R / len(sample)
        rows["moe:%s" % ("gate_up" if what == "up" else "down")] = {
            "us_per_call": round(ms * 1e3, 2), "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
            "tflops": round(fl / (ms / 1e3) / 1e12, 1), "frac_fp8_peak": round(fl / (ms / 1e3) / 1e12 / fp8, 3),
            "bound": "hbm (roofline max(%.1f us flops, %.1f us bytes))" % (fl / fp8 / 1e6, nbytes / hbm / 1e3),
            "cpu_oracle": oracle_row(nbytes, ot, 1e9, "GB/s",
                                     "the first row of every non-empty expert (%d rows), time scaled to %d rows"
                                     % (len(sample), R))}
    del moe, qa, sa, qw, sw, y

    # --- whole-model recalibration (32 layers x 4 weights, power-of-2 scales, one call)
    tensors = []
    for _, _, w in wl.model_weights_after_step(device=dev):
        N, K = w.shape
        tensors.append((w, torch.empty((N, K), dtype=torch.uint8, device=dev),
                        torch.empty((N // 128, K // 128), dtype=torch.float32, device=dev)))
    nbytes = sum(recal_bytes(*w.shape) for w, _, _ in tensors)
    ms = graph_ms([lambda: fq.recalibrate(tensors, fq.SCALE_POW2)] * 3)
    gbs = nbytes / (ms / 1e3) / 1e9
    ow = bits(tensors[1][0])           # one O-projection weight, 4096 x 4096
    t0 = time.perf_counter()
    oracle.quant_weight(ow, 1)
    ot = (time.perf_counter() - t0) * nbytes / recal_bytes(*ow.shape)
    rows["recalibrate:model_pow2"] = {
        "ms": round(ms, 3), "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3), "tensors": len(tensors),
        "params": int(sum(w.numel() for w, _, _ in tensors)),
        "cpu_oracle": oracle_row(nbytes, ot, 1e9, "GB/s",
                                 "one 4096x4096 weight, time scaled to the whole model's bytes")}
    # per-step overhead proxy: the model's recalibration against 3 x 32 layers of
    # the step's forward GEMMs (forward + the two backward GEMMs of a training step)
    rows["recal_overhead"] = {
        "value": round(ms / (3 * wl.LLAMA8B_LAYERS * gemm_ms_step), 4),
        "definition": "recalibrate:model_pow2 ms / (3 x 32 x the benchmark step's four GEMM ms)",
        "context": "the pages report about 2-3% recalibration overhead per training step on H100"}
    del tensors
    torch.cuda.empty_cache()
    return rows


def max_over_ranks(value, device):
    """The maximum of a per-rank float over all ranks (identity for one rank):
    the job's time is its slowest replica's."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(work_per_step, steps, world, secs):
    """Whole-job rate: every replica processes work_per_step per step; secs is
    the slowest replica's time for `steps` steps."""
    return world * work_per_step * steps / secs


def ours(args):
    import torch.distributed as dist
    import fp8_block_scaled_fp8bq_b200 as fq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local)
    fq.lib()

    def rank_sync():
        if world > 1:
            dist.barrier()

    step = LayerStep(fq, device)
    with ClockSampler(local) as clk:
        secs, events = timed_steps(step, args.steps, args.warmup, rank_sync)
    secs = max_over_ranks(secs, device)
    K = args.steps
    flops = gemm_flops_step()
    value = job_throughput(flops, K, world, secs) / 1e12

    # per-row figures from the per-launch events
    def avg_ms(key):
        return sum(a.elapsed_time(b) for a, b in events[key]) / len(events[key])

    peaks = load_peaks()
    sustained = secs > 1.0
    bf16_peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    fp8_peak = 2.0 * bf16_peak
    rows = {}
    gemm_ms_total = 0.0
    for name, (N, K_) in wl.LLAMA8B_SHAPES.items():
        ms = avg_ms("gemm:" + name)
        gemm_ms_total += ms
        tf = 2.0 * M_TOKENS * N * K_ / (ms / 1e3) / 1e12
        rows["gemm:" + name] = {"ms": round(ms, 4), "tflops": round(tf, 1), "frac_fp8_peak": round(tf / fp8_peak, 3)}
        qms = avg_ms("quant_act:" + name)
        gbs = quant_act_bytes(M_TOKENS, K_) / (qms / 1e3) / 1e9
        rows["quant_act:" + name] = {"ms": round(qms, 4), "gbs": round(gbs, 1),
                                     "frac_hbm": round(gbs / peaks["hbm_gbs"], 3)}
    rms = avg_ms("recalibrate")
    rb = sum(recal_bytes(N, K_) for N, K_ in wl.LLAMA8B_SHAPES.values())
    rows["recalibrate:layer"] = {"ms": round(rms, 4), "gbs": round(rb / (rms / 1e3) / 1e9, 1),
                                 "frac_hbm": round(rb / (rms / 1e3) / 1e9 / peaks["hbm_gbs"], 3)}
    achieved = flops / (gemm_ms_total / 1e3) / 1e12
    traffic = committed_traffic()
    roofline = {"bound": "tensor", "kernel": "gemm_promote_kernel (4 launches per step, averaged)",
                "achieved": round(achieved, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / fp8_peak, 4), "traffic": traffic,
                "peak_note": "%s bf16 %s x 2 (nominal fp8:bf16 ratio)" % (
                    "of measured" if peaks["source"] == "measured" else "of fallback",
                    "sustained" if sustained else "burst")}

    # end to end: host buffers, copies inside the timed region
    Ke = max(1, min(K, 10))
    e2e_s, h2d, d2h = e2e_steps(fq, step, Ke, rank_sync)
    e2e_s = max_over_ranks(e2e_s, device)
    e2e = {"value": round(job_throughput(flops, Ke, world, e2e_s) / 1e12, 2), "unit": "TFLOP/s",
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": Ke}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(secs / K * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 x e4m3 -> f32 accumulate, bf16 out",
            "data": "synthetic (seeded; Llama-3.1-8B shapes, no model weights)",
            "config": {"workload": WORKLOAD, "tokens": M_TOKENS,
                       "shapes_NK": {n: list(s) for n, s in wl.LLAMA8B_SHAPES.items()}, "scale_mode": "fp32",
                       "l2": "inputs larger than L2 (about 2 GB touched per step vs 126 MB L2); no flush",
                       "parallelism": "replicas" if world > 1 else "single gpu"},
            "roofline": roofline, "rows": rows, "e2e": e2e,
            "gpu_launches": LAUNCHES_PER_STEP * K, "clocks": clk.summary(),
        }
        if world == 1:
            line["cpu_baseline"] = cpu_baseline_oracle()
            if not args.step_only:
                rows.update(config_rows(fq, device, peaks, gemm_ms_total))
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def reference(args):
    """The oracle as it stands, on the host cores, K steps of a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    R = max(1, min(32, oracle.num_threads()))
    data = []
    for i, (name, (N, K)) in enumerate(wl.LLAMA8B_SHAPES.items()):
        x = wl.activations(R, K, seed=100 + i).view(torch.int16).numpy().view(np.uint16)
        # the weight sample: 128-row block rows of W (all of K), enough for every thread
        nrows = min(N, 128 * max(1, min(8, R // 2)))
        w = wl.weights(nrows, K, seed=200 + i).view(torch.int16).numpy().view(np.uint16)
        data.append((x, w, N, K, nrows))

    def one_step():
        flops = 0.0
        for x, w, N, K, nrows in data:
            qw, sw = oracle.quant_weight(w, 0)
            qa, sa = oracle.quant_act(x, 0)
            oracle.gemm(qa, sa, qw, sw)
            flops += 2.0 * x.shape[0] * nrows * K
        return flops

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    flops = 0.0
    for _ in range(args.steps):
        flops += one_step()
    secs = time.perf_counter() - t0
    value = flops / secs / 1e12
    sample = ("per step: %d rows of each linear's input (1x128 quant) times a %d-row block of its weight "
              "(128x128 quant + FP64 GEMM)" % (R, data[0][4]))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic", "config": {"workload": WORKLOAD, "tokens": M_TOKENS},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


CASES = (["gemm:" + n for n in NAMES] + ["decode:" + n for n in NAMES] + ["cublas:" + n for n in NAMES] +
         ["quant_act:4096", "quant_act:14336", "recalibrate:layer", "quant_weight:gate_up", "moe:up", "moe:down",
          "swiglu:gate_up", "moe_swiglu:up", "adamw_recal:layer", "quant_act_t:4096", "quant_act_t:14336",
          "transpose_weight:gate_up", "prefill_attn:4x2048", "prefill_attn:1x2048", "prefill_attn:1x8192",
          "decode_attn:1x32768", "decode_attn:16x8192", "decode_attn:64x4096",
          "decode_attn:256x2048", "recalibrate:model"] + ["dgrad:" + n for n in NAMES] +
         ["wgrad:" + n for n in NAMES])


def prefill_attn_flops(B, S, Hq, D=128):
    """Causal attention: 2 x 2 x D FLOPs per (query, visible key, head)."""
    return 4.0 * D * (S * (S + 1) // 2) * Hq * B


def prefill_attn_inputs(fq, B, S, dev, Hq=32, Hkv=8):
    """Seeded bf16 Q, K, V ~ N(0, 1) quantized 1x128 per head vector on the GPU."""
    g = torch.Generator(device=dev).manual_seed(17)
    q = torch.randn((B * S * Hq, 128), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((B * S * Hkv, 128), generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn((B * S * Hkv, 128), generator=g, device=dev).to(torch.bfloat16)
    qq, qs = fq.quant_act(q)
    kq, ks = fq.quant_act(k)
    vq, vs = fq.quant_act(v)
    shape_q, shape_kv = (B, S, Hq), (B, S, Hkv)
    lens = torch.full((B,), S, dtype=torch.int32, device=dev)
    return ((qq.view(*shape_q, 128), qs[0, :B * S * Hq].contiguous().view(shape_q)),
            kq.view(*shape_kv, 128), ks[0, :B * S * Hkv].contiguous().view(shape_kv),
            vq.view(*shape_kv, 128), vs[0, :B * S * Hkv].contiguous().view(shape_kv), lens)


def decode_bytes(M, N, K):
    """Weight codes + weight scales + bf16 activations in + bf16 out."""
    return N * K + ((N + 127) // 128) * (K // 128) * 4 + M * K * 2 + M * N * 2


def moe_bytes(R, E, N, K):
    """Expert weights + activation codes/scales + bf16 out (each read once)."""
    return E * N * K + E * (N // 128) * (K // 128) * 4 + R * K + R * (K // 128) * 4 + R * N * 2


def run_case(args):
    """One kernel on one shape, for profiling (ncu) and per-kernel timing: --warmup
    untimed launches, then --steps timed launches; prints a JSON line with the
    average launch time.  Not the benchmark line."""
    import fp8_block_scaled_fp8bq_b200 as fq
    fq.lib()
    M = args.tokens
    kind, what = args.case.split(":")
    dev = torch.device("cuda", 0)
    mode = fq.SCALE_POW2 if args.pow2 else fq.SCALE_FP32
    if kind == "gemm":
        N, K = wl.LLAMA8B_SHAPES[what]
        x = wl.activations(M, K, seed=1, device=dev)
        w = wl.weights(N, K, seed=2, device=dev)
        qa, sa = fq.quant_act(x, mode)
        qw, sw = fq.quant_weight(w, mode)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        variant = (fq.GEMM_NATIVE_POW2 if args.native else fq.GEMM_PROMOTE_PAIR if args.pair
                   else fq.GEMM_PROMOTE_PAIR_N128 if args.pair128 else fq.GEMM_PROMOTE)
        fn = lambda: fq.gemm(qa, sa, qw, sw, mode, out=y, variant=variant)  # noqa: E731
        work, unit = 2.0 * M * N * K / 1e12, "TFLOP/s"
    elif kind == "cublas":
        # context only: cuBLASLt FP8 GEMM through torch._scaled_mm on the same shape
        # (per-tensor scales; blockwise scales if this torch build accepts them)
        N, K = wl.LLAMA8B_SHAPES[what]
        a = wl.activations(M, K, seed=1, device=dev).to(torch.float8_e4m3fn)
        b = wl.weights(N, K, seed=2, device=dev).mul(20).to(torch.float8_e4m3fn)
        sa_ = torch.ones((), dtype=torch.float32, device=dev)
        sb_ = torch.ones((), dtype=torch.float32, device=dev)
        if args.pow2:
            # blockwise: 1x128 for a (outer-dim-major), 128x128 for b; the layouts
            # torch documents in its error text; fall back to per-tensor if refused
            cand_a = torch.ones((K // 128, M), dtype=torch.float32, device=dev).t()
            for cand_b in (torch.ones(((N + 127) // 128, K // 128), dtype=torch.float32, device=dev).t(),
                           torch.ones((K // 128, (N + 127) // 128), dtype=torch.float32, device=dev)):
                try:
                    torch._scaled_mm(a, b.t(), scale_a=cand_a, scale_b=cand_b, out_dtype=torch.bfloat16)
                    sa_, sb_ = cand_a, cand_b
                    print(json.dumps({"case": args.case, "cublas_scaling": "blockwise 1x128 x 128x128"}))
                    break
                except RuntimeError as e:
                    print(json.dumps({"case": args.case, "cublas_refused": str(e).splitlines()[0][:120]}))
        fn = lambda: torch._scaled_mm(a, b.t(), scale_a=sa_, scale_b=sb_, out_dtype=torch.bfloat16)  # noqa: E731
        work, unit = 2.0 * M * N * K / 1e12, "TFLOP/s"
    elif kind == "decode":
        N, K = wl.LLAMA8B_SHAPES[what]
        x = wl.activations(M, K, seed=1, device=dev)
        w = wl.weights(N, K, seed=2, device=dev)
        qw, sw = fq.quant_weight(w, mode)
        del w
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(max(256, fq.gemm_decode_workspace_size(M, N, K)), dtype=torch.uint8, device=dev)
        # successive calls read different copies of the weight (none finds it in L2)
        qws = itertools.cycle([qw] + [qw.clone() for _ in range(rotations(N * K) - 1)])
        fn = lambda: fq.gemm_decode(x, next(qws), sw, mode, out=y, ws=ws)  # noqa: E731
        work, unit = decode_bytes(M, N, K) / 1e9, "GB/s"
    elif kind == "moe":
        moe = wl.moe_layer(seed=0, device=dev)
        x, w = moe["x_" + what], moe["w_" + what]
        E, N, K = w.shape
        R = x.shape[0]
        qa, sa = fq.quant_act(x, mode)
        qw, sw = fq.quant_weight(w.reshape(E * N, K), mode)
        qw, sw = qw.view(E, N, K), sw.view(E, N // 128, K // 128)
        off = moe["offsets"].to(torch.int32).to(dev)
        y = torch.empty((R, N), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.grouped_gemm(qa, sa, qw, sw, off, mode, out=y)  # noqa: E731
        work, unit = moe_bytes(R, E, N, K) / 1e9, "GB/s"
        print(json.dumps({"case": args.case, "flops": 2.0 * R * N * K}))
    elif kind == "swiglu":
        # fused gate+up: the Llama gate+up weight [2I, K] taken as interleaved,
        # H codes [M, I] and scales out (no bf16 H)
        N, K = wl.LLAMA8B_SHAPES[what]
        x = wl.activations(M, K, seed=1, device=dev)
        w = wl.weights(N, K, seed=2, device=dev)
        qa, sa = fq.quant_act(x, mode)
        qw, sw = fq.quant_weight(w, mode)
        qh = torch.empty((M, N // 2), dtype=torch.uint8, device=dev)
        sh = torch.empty(fq.act_scale_shape(M, N // 2), dtype=torch.float32, device=dev)
        fn = lambda: fq.gemm_swiglu_quant(qa, sa, qw, sw, mode, qh=qh, sh=sh)  # noqa: E731
        work, unit = 2.0 * M * N * K / 1e12, "TFLOP/s"
    elif kind == "moe_swiglu":
        moe = wl.moe_layer(seed=0, device=dev)
        x, w = moe["x_" + what], moe["w_" + what]
        E, N, K = w.shape
        R = x.shape[0]
        qa, sa = fq.quant_act(x, mode)
        qw, sw = fq.quant_weight(w.reshape(E * N, K), mode)
        qw, sw = qw.view(E, N, K), sw.view(E, N // 128, K // 128)
        off = moe["offsets"].to(torch.int32).to(dev)
        qh = torch.empty((R, N // 2), dtype=torch.uint8, device=dev)
        sh = torch.empty(fq.act_scale_shape(R, N // 2), dtype=torch.float32, device=dev)
        fn = lambda: fq.grouped_gemm_swiglu_quant(qa, sa, qw, sw, off, mode, qh=qh, sh=sh)  # noqa: E731
        # bytes: A codes + scales, W codes + scales, H codes + scales
        work = (R * K + 4 * R * (K // 128) + E * N * K + 4 * E * (N // 128) * (K // 128) + R * N // 2
                + 4 * R * (N // 256)) / 1e9
        unit = "GB/s"
        print(json.dumps({"case": args.case, "flops": 2.0 * R * N * K}))
    elif kind == "decode_attn":
        # Llama-3.1-8B attention (32 query heads, 8 key/value heads, D = 128):
        # one query token per sequence over a full FP8 cache of the given length
        B_, S_ = (int(v) for v in what.split("x"))
        Hq, Hkv = 32, 8
        g = torch.Generator(device=dev).manual_seed(5)
        kq = torch.randint(0, 0x7E, (B_, S_, Hkv, 128), generator=g, device=dev, dtype=torch.uint8)
        vq = torch.randint(0, 0x7E, (B_, S_, Hkv, 128), generator=g, device=dev, dtype=torch.uint8)
        kq |= torch.randint(0, 2, kq.shape, generator=g, device=dev, dtype=torch.uint8) << 7
        vq |= torch.randint(0, 2, vq.shape, generator=g, device=dev, dtype=torch.uint8) << 7
        ks = torch.rand((B_, S_, Hkv), generator=g, device=dev) * 0.01 + 0.001
        vs = torch.rand((B_, S_, Hkv), generator=g, device=dev) * 0.01 + 0.001
        qv = torch.randn((B_, Hq, 128), generator=g, device=dev).to(torch.bfloat16)
        lens = torch.full((B_,), S_, dtype=torch.int32, device=dev)
        out = torch.empty((B_, Hq, 128), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(16, int(fq.lib().fp8bq_decode_attention_workspace_size(B_, Hq, Hkv, S_))),
                         dtype=torch.uint8, device=dev)
        fn = lambda: fq.decode_attention(qv, kq, ks, vq, vs, lens, out=out, ws=ws)  # noqa: E731
        work = (B_ * S_ * Hkv * (2 * 128 + 8) + 2 * B_ * Hq * 128 * 2) / 1e9
        unit = "GB/s"
    elif kind == "prefill_attn":
        # Llama-3.1-8B attention (32 query heads, 8 key/value heads, D = 128),
        # causal over B sequences of S tokens, FP8 queries, keys and values
        B_, S_ = (int(v) for v in what.split("x"))
        q, kq, ks, vq, vs, lens = prefill_attn_inputs(fq, B_, S_, dev)
        out = torch.empty((B_, S_, 32, 128), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.prefill_attention(*q, kq, ks, vq, vs, lens, out=out)  # noqa: E731
        work, unit = prefill_attn_flops(B_, S_, 32) / 1e12, "TFLOP/s"
    elif kind == "quant_act_t":
        K = int(what)
        x = wl.activations(M, K, seed=1, device=dev)
        qt = torch.empty((K, M), dtype=torch.uint8, device=dev)
        st = torch.empty((fq.ceil_div(M, 128), K), dtype=torch.float32, device=dev)
        fn = lambda: fq.quant_act_t(x, mode, qt=qt, st=st)  # noqa: E731
        work, unit = quant_act_bytes(M, K) / 1e9, "GB/s"
    elif kind == "transpose_weight":
        N, K = wl.LLAMA8B_SHAPES[what]
        q, sw = fq.quant_weight(wl.weights(N, K, seed=2, device=dev), mode)
        qt = torch.empty((K, N), dtype=torch.uint8, device=dev)
        swt = torch.empty((sw.shape[1], sw.shape[0]), dtype=torch.float32, device=dev)
        fn = lambda: fq.transpose_weight(q, sw, qt=qt, swt=swt)  # noqa: E731
        work, unit = 2.0 * N * K / 1e9, "GB/s"
    elif kind == "dgrad":
        # dX [M, K] = dY [M, N] . W [N, K] through W^T's codes
        N, K = wl.LLAMA8B_SHAPES[what]
        dy = wl.activations(M, N, seed=1, device=dev)
        q_dy, s_dy = fq.quant_act(dy, mode)
        qwt, swt = fq.transpose_weight(*fq.quant_weight(wl.weights(N, K, seed=2, device=dev), mode))
        dx = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.gemm_dgrad(q_dy, s_dy, qwt, swt, mode, out=dx)  # noqa: E731
        work, unit = 2.0 * M * N * K / 1e12, "TFLOP/s"
    elif kind == "wgrad":
        # dW [N, K] = dY^T X over M tokens
        N, K = wl.LLAMA8B_SHAPES[what]
        qa, sa = fq.quant_act_t(wl.activations(M, N, seed=1, device=dev), mode)
        qb, sb = fq.quant_act_t(wl.activations(M, K, seed=2, device=dev), mode)
        dw = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.gemm_wgrad(qa, sa, qb, sb, M, mode, out=dw)  # noqa: E731
        work, unit = 2.0 * M * N * K / 1e12, "TFLOP/s"
    elif kind == "adamw_recal":
        # AdamW on fp32 master weights + moments of the four Llama-8B-shaped
        # linears, fused with the bf16 copy and the 128x128 recalibration
        tensors = []
        nbytes = 0
        for i, (N, K) in enumerate(wl.LLAMA8B_SHAPES.values()):
            g = torch.Generator(device=dev).manual_seed(300 + i)
            p = torch.randn((N, K), generator=g, device=dev) * 0.02
            gr = torch.randn((N, K), generator=g, device=dev) * 1e-3
            m = torch.randn((N, K), generator=g, device=dev) * 1e-4
            v = torch.rand((N, K), generator=g, device=dev) * 1e-6
            w = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
            q = torch.empty((N, K), dtype=torch.uint8, device=dev)
            s_ = torch.empty(((N + 127) // 128, (K + 127) // 128), dtype=torch.float32, device=dev)
            tensors.append((p, gr, m, v, w, q, s_))
            # read p, g, m, v; write p, m, v, w, q, scales
            nbytes += N * K * (16 + 12 + 2 + 1) + 4 * ((N + 127) // 128) * ((K + 127) // 128)
        fn = lambda: fq.adamw_recalibrate(tensors, lr=1e-5, beta1=0.9, beta2=0.95, eps=1e-8,  # noqa: E731
                                          weight_decay=0.1, step=100, mode=mode)
        work, unit = nbytes / 1e9, "GB/s"
    elif kind == "quant_act":
        K = int(what)
        x = wl.activations(M, K, seed=1, device=dev)
        q = torch.empty((M, K), dtype=torch.uint8, device=dev)
        sa = torch.empty(fq.act_scale_shape(M, K), dtype=torch.float32, device=dev)
        fn = lambda: fq.quant_act(x, mode, q=q, sa=sa)  # noqa: E731
        work, unit = quant_act_bytes(M, K) / 1e9, "GB/s"
    elif kind == "quant_weight":
        N, K = wl.LLAMA8B_SHAPES[what]
        w = wl.weights(N, K, seed=2, device=dev)
        q = torch.empty((N, K), dtype=torch.uint8, device=dev)
        sw = torch.empty((fq.ceil_div(N, 128), fq.ceil_div(K, 128)), dtype=torch.float32, device=dev)
        fn = lambda: fq.quant_weight(w, mode, q=q, sw=sw)  # noqa: E731
        work, unit = recal_bytes(N, K) / 1e9, "GB/s"
    elif what == "model":
        # the whole model's recalibration: 32 layers x 4 weights after one
        # synthetic update, one call (128 tensors)
        tensors = []
        for _, _, w in wl.model_weights_after_step(device=dev):
            N, K = w.shape
            tensors.append((w, torch.empty((N, K), dtype=torch.uint8, device=dev),
                            torch.empty((fq.ceil_div(N, 128), fq.ceil_div(K, 128)), dtype=torch.float32,
                                        device=dev)))
        fn = lambda: fq.recalibrate(tensors, mode)  # noqa: E731
        work, unit = sum(recal_bytes(*w.shape) for w, _, _ in tensors) / 1e9, "GB/s"
    else:
        step = LayerStep(fq, dev, mode=mode)
        fn = lambda: fq.recalibrate(step.recal_list, mode)  # noqa: E731
        work, unit = sum(recal_bytes(N, K) for N, K in wl.LLAMA8B_SHAPES.values()) / 1e9, "GB/s"
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if args.graph:
        # launch-bound cases: capture the launches in a CUDA graph so the host
        # does not pace the GPU; one replay runs --steps calls
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(args.steps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        t0.record()
        g.replay()
        t1.record()
    else:
        t0.record()
        for _ in range(args.steps):
            fn()
        t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / args.steps
    print(json.dumps({"case": args.case, "tokens": M, "pow2": bool(args.pow2), "graph": bool(args.graph),
                      "launches": args.steps,
                      "ms_per_launch": round(ms, 5), "rate": round(work / (ms / 1e3), 1), "unit": unit}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=CASES, default=None,
                    help="time one kernel on one shape instead of the benchmark step (for profiling)")
    ap.add_argument("--tokens", type=int, default=M_TOKENS, help="M for --case")
    ap.add_argument("--pow2", action="store_true", help="power-of-2 scales for --case")
    ap.add_argument("--graph", action="store_true", help="--case: time a CUDA graph of --steps calls")
    ap.add_argument("--native", action="store_true", help="--case gemm with --pow2: native block-scaled MMA")
    ap.add_argument("--pair", action="store_true", help="--case gemm: the CTA-pair promotion kernel")
    ap.add_argument("--pair128", action="store_true",
                    help="--case gemm: the CTA-pair promotion kernel with 256x128 tiles")
    ap.add_argument("--step-only", action="store_true",
                    help="only the benchmark step (no rows for the other workload configurations)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.case:
        run_case(args)
    elif args.impl == "reference":
        reference(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
