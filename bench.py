"""Benchmark of the FP8 runtime linear path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference] [--no-extras]

One step = one pass of the hot path over one batch: fp8_quantize of the bf16
activations X (amax reduce, scale, RNE cast) and fp8_scaled_gemm with the
pre-quantised static weight (tcgen05 MMA, FP32 accumulation, scaled BF16
epilogue) -- exactly what fp8_linear_forward does in one call.

Default workload ``llama70b_prefill``: X [4096, 8192] per-token scales, W
[28672, 8192] per-output-channel scales, E4M3, Y [4096, 28672] bf16.  ``value``
is FP8 GEMM TFLOP/s of the whole step (2*M*N*K per step / step time); every
step moves ~534 MB (> the 126 MB L2), so no extra L2 flush is needed.

Extras (rank 0, N=1): the 64 Mi-element quantize sweep in GB/s for E4M3 and
E5M2 (codes + scale + dequant), the block-scaled and MXFP8 GEMMs, the delayed
per-tensor linear step and the small per-tensor linear latency.

Multi-GPU: one process per GPU, each runs the same step on its own batch
(weak scaling, no data-path collective); time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import threading
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantize GB/s and FP8 scaled-GEMM TFLOPS (1 B200), as % of HBM/FP8 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 2.0          # nominal dense ratio (4.5 / 2.25 PFLOP/s)
WORKLOADS = {
    "llama70b_prefill": dict(M=4096, K=8192, N=28672, x_mode=1, w_mode=1),
    # the same layer at decode: 16 tokens per call (the weight-streaming kernel)
    "llama70b_decode": dict(M=16, K=8192, N=28672, x_mode=1, w_mode=1),
    "block_scaled": dict(M=8192, K=8192, N=28672, x_mode=2, w_mode=3),
    "mx": dict(M=16384, K=8192, N=8192, x_mode=4, w_mode=4),
}


def max_over_ranks(value_ms: float, dist=None, device="cpu") -> float:
    """The job's time is the slowest rank's (device-timed) time."""
    if dist is None:
        return value_ms
    import torch
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Aggregate throughput of `world` ranks that each processed `units_per_rank` in `ms`."""
    return world * units_per_rank / (ms * 1e-3)


def rank_batch(x: np.ndarray, rank: int) -> np.ndarray:
    """Each rank's own batch (weak scaling): the seeded batch, rows rotated by rank."""
    return np.roll(x, rank, axis=0) if rank else x


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_digest():
    h = hashlib.sha256()
    for fn in ("gemm_sm100.cu", "gemm_common.cuh", "decode_sm100.cu", "quantize.cu", "ptx.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "fp8_dynamic_scaled_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def use_sustained_peak(timed_ms: float, clocks: dict):
    """The roofline denominator follows the run: the sustained (power-capped) FP8 figure
    only when the timed region lasted at least 1 s and the sampled clocks saw the power
    cap, else the burst figure.  Returns (use the sustained figure, power cap seen)."""
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    return timed_ms >= 1000.0 and capped, capped


def profiled_traffic(kernel_tag: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel sources (the summary records the source digest)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    digest = source_digest()
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and parts[0] == kernel_tag and parts[1] == digest:
                return float(parts[2])
    return None


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.reader = None

    def _read(self):
        for line in self.proc.stdout:
            if line.strip():
                self.lines.append(line)

    def _wait_lines(self, n: int, limit_s: float):
        t0 = time.monotonic()
        while len(self.lines) < n and time.monotonic() - t0 < limit_s and self.proc.poll() is None:
            time.sleep(0.01)

    def __enter__(self):
        # the sampler is live (its first sample read) before the timed region starts, and
        # one more sample is read after it ends, so that a region shorter than the 200 ms
        # period still has samples on both sides
        self.lines = []
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        self._wait_lines(1, 5.0)
        return self

    def __exit__(self, *exc):
        if self.proc is None:
            return
        self._wait_lines(len(self.lines) + 1, 1.0)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait()
        self.reader.join(timeout=5)
        self.lines = list(self.lines)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            p = [x.strip() for x in l.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx = float(p[2])
            except ValueError:
                continue
            for name, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- helpers
def to_dev_bf16(torch, u16):
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def make_workload(torch, fp8, name, rank):
    """Inputs for one rank (seeded; rank 0 gets the reference seed), W quantised once."""
    from fp8_dynamic_scaled_b200 import inputs
    wl = WORKLOADS[name]
    M, K, N = wl["M"], wl["K"], wl["N"]
    if name in ("llama70b_prefill", "llama70b_decode"):
        x, w = inputs.llama70b_prefill(M, K, N)
    elif name == "block_scaled":
        x, w = inputs.block_scaled(M, K, N)
    else:
        x, w = inputs.mx_delayed(M, K, N)
    x = rank_batch(x, rank)
    xd = to_dev_bf16(torch, x)
    wd = to_dev_bf16(torch, w)
    wq, ws, _ = fp8.empty_quant_outputs(N, K, wl["w_mode"])
    fp8.fp8_quantize(wd, fp8.FP8_E4M3, wl["w_mode"], wq, ws, workspace=fp8.workspace_for(0, N, 0, K, wl["w_mode"]))
    torch.cuda.synchronize()
    del wd
    return dict(M=M, K=K, N=N, x_mode=wl["x_mode"], w_mode=wl["w_mode"], x=xd, x_host=x, wq=wq, ws=ws)


def quantize_launches(mode):
    return 2 if mode in (0, 5) else 1


def time_linear_steps(torch, fp8, wl, steps, warmup, stream, barrier=None):
    """Device-timed K steps of quantize(X) -> scaled GEMM; per-kernel events on the stream."""
    M, K, N, xm, wm = wl["M"], wl["K"], wl["N"], wl["x_mode"], wl["w_mode"]
    xq, xs, _ = fp8.empty_quant_outputs(M, K, xm)
    qws = fp8.workspace_for(0, M, 0, K, xm)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        fp8.fp8_quantize(wl["x"], fp8.FP8_E4M3, xm, xq, xs, dev_status=status, workspace=qws, stream=stream)
        if evs:
            evs[1].record(stream)
        fp8.fp8_scaled_gemm(xq, xs, xm, fp8.FP8_E4M3, wl["wq"], wl["ws"], wm, fp8.FP8_E4M3, y, dev_status=status,
                            stream=stream)
        if evs:
            evs[2].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if barrier:
        barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(steps):
            step(evs[i])
        end.record(stream)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    total_ms = start.elapsed_time(end)
    q_ms = [e[0].elapsed_time(e[1]) for e in evs]
    g_ms = [e[1].elapsed_time(e[2]) for e in evs]
    st = int(status.item())
    if st != 0:
        raise RuntimeError(f"device status {fp8.fp8_status_string(st)} during the timed steps")
    return total_ms, q_ms, g_ms, y


def time_e2e(torch, fp8, wl, steps, warmup, stream):
    """The step through the public call with host buffers: every step copies its X from
    pinned host memory to the device, runs fp8_linear_forward and copies its Y back to
    pinned host memory, all inside the timed region.  The copies run on their own
    streams with two device buffers of X and Y, so step i+1's upload and step i's
    download overlap each other and the compute (PCIe carries both directions at once);
    events order each buffer's reuse."""
    M, K, N, xm, wm = wl["M"], wl["K"], wl["N"], wl["x_mode"], wl["w_mode"]
    x_pin = torch.from_numpy(np.ascontiguousarray(wl["x_host"]).view(np.int16)).view(torch.bfloat16).pin_memory()
    y_pin = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xd = [torch.empty((M, K), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    yd = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    ws = fp8.workspace_for(2, M, N, K, xm)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def run(n):
        for i in range(n):
            b = i % 2
            if i >= 2:
                s_in.wait_event(comp_done[b])          # step i-2 has consumed xd[b]
            with torch.cuda.stream(s_in):
                xd[b].copy_(x_pin, non_blocking=True)
                h2d_done[b].record(s_in)
            stream.wait_event(h2d_done[b])
            if i >= 2:
                stream.wait_event(d2h_done[b])         # step i-2's Y has left yd[b]
            fp8.fp8_linear_forward(xd[b], fp8.FP8_E4M3, xm, wl["wq"], wl["ws"], wm, fp8.FP8_E4M3, yd[b], ws,
                                   stream=stream)
            comp_done[b].record(stream)
            s_out.wait_event(comp_done[b])
            with torch.cuda.stream(s_out):
                y_pin[b].copy_(yd[b], non_blocking=True)
                d2h_done[b].record(s_out)

    run(warmup)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    s_in.wait_event(start)
    s_out.wait_event(start)
    run(steps)
    stream.wait_stream(s_out)
    end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    return ms, x_pin.numel() * 2, y_pin[0].numel() * 2


def time_kernel(torch, fn, reps, stream, warmup=3):
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for a, b in evs:
            a.record(stream)
            fn()
            b.record(stream)
    torch.cuda.synchronize()
    ts = sorted(a.elapsed_time(b) for a, b in evs)
    return statistics.median(ts), ts[min(len(ts) - 1, int(0.95 * len(ts)))]


def extras(torch, fp8, stream, peaks, gpu_index=0):
    """Per-config numbers behind the metric (rank 0, one GPU)."""
    from fp8_dynamic_scaled_b200 import inputs
    out = {}
    hbm = peaks["hbm_gbs"]
    # quantize sweep, 64 Mi elements, per-tensor current scaling, codes + scale + dequant
    xs = to_dev_bf16(torch, inputs.quant_sweep())
    rows, cols = xs.shape
    q, s, d = fp8.empty_quant_outputs(rows, cols, fp8.FP8_SCALE_TENSOR, dequant=True)
    ws = fp8.workspace_for(0, rows, 0, cols, fp8.FP8_SCALE_TENSOR)
    nbytes = rows * cols * (2 + 1 + 2) + 4
    for name, fmt in (("e4m3", fp8.FP8_E4M3), ("e5m2", fp8.FP8_E5M2)):
        med, p95 = time_kernel(torch, lambda: fp8.fp8_quantize(xs, fmt, fp8.FP8_SCALE_TENSOR, q, s, dequant=d,
                                                               workspace=ws, stream=stream), 20, stream)
        out[f"quant_sweep_{name}"] = {"us_median": med * 1e3, "us_p95": p95 * 1e3, "algorithmic_bytes": nbytes,
                                      "GB_per_s": nbytes / (med * 1e-3) / 1e9,
                                      "frac_of_hbm": nbytes / (med * 1e-3) / 1e9 / hbm}
    # codes only (no dequant)
    med, _ = time_kernel(torch, lambda: fp8.fp8_quantize(xs, fp8.FP8_E4M3, fp8.FP8_SCALE_TENSOR, q, s, workspace=ws,
                                                         stream=stream), 20, stream)
    nb = rows * cols * 3 + 4
    out["quant_sweep_e4m3_codes_only"] = {"us_median": med * 1e3, "GB_per_s": nb / (med * 1e-3) / 1e9,
                                          "frac_of_hbm": nb / (med * 1e-3) / 1e9 / hbm}
    del xs, q, s, d
    torch.cuda.empty_cache()
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    for name in ("block_scaled", "mx"):
        wl = make_workload(torch, fp8, name, 0)
        M, K, N = wl["M"], wl["K"], wl["N"]
        total, qms, gms, _ = time_linear_steps(torch, fp8, wl, 10, 3, stream)
        g = statistics.median(gms)
        qm = statistics.median(qms)
        xbytes = M * K * 3 + (M * (K // 32) if wl["x_mode"] == 4 else 4 * M * (-(-K // 128)))
        out[name] = {"gemm_us_median": g * 1e3, "gemm_tflops": 2 * M * N * K / (g * 1e-3) / 1e12,
                     "gemm_frac_of_fp8_peak_burst": 2 * M * N * K / (g * 1e-3) / 1e12 / fp8_peak,
                     "x_quantize_us": qm * 1e3, "x_quantize_GB_per_s": xbytes / (qm * 1e-3) / 1e9,
                     "step_ms": total / 10}
        del wl
        torch.cuda.empty_cache()
    # delayed per-tensor scaling: 16 steps of the drifting sequence (MX-config shapes)
    M, K, N = 16384, 8192, 8192
    base = inputs.delayed_base(M, K)
    xs_steps = [to_dev_bf16(torch, inputs.delayed_step_input(t, M, K, base=base)) for t in range(4)]
    _, w = inputs.mx_delayed(M, K, N)
    wq, wsc, _ = fp8.empty_quant_outputs(N, K, fp8.FP8_SCALE_TENSOR)
    fp8.fp8_quantize(to_dev_bf16(torch, w), fp8.FP8_E4M3, fp8.FP8_SCALE_TENSOR, wq, wsc,
                     workspace=fp8.workspace_for(0, N, 0, K, fp8.FP8_SCALE_TENSOR))
    hist = fp8.History(16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    lws = fp8.workspace_for(2, M, N, K, fp8.FP8_SCALE_DELAYED)
    xq, xsc, _ = fp8.empty_quant_outputs(M, K, fp8.FP8_SCALE_DELAYED)
    qws = fp8.workspace_for(0, M, 0, K, fp8.FP8_SCALE_DELAYED)
    times_q, times_l = [], []
    for t in range(16):
        x = xs_steps[t % 4]
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        with torch.cuda.stream(stream):
            a.record(stream)
            fp8.fp8_quantize(x, fp8.FP8_E4M3, fp8.FP8_SCALE_DELAYED, xq, xsc, hist=hist, workspace=qws, stream=stream)
            b.record(stream)
            fp8.fp8_scaled_gemm(xq, xsc, fp8.FP8_SCALE_TENSOR, fp8.FP8_E4M3, wq, wsc, fp8.FP8_SCALE_TENSOR,
                                fp8.FP8_E4M3, y, stream=stream)
            c.record(stream)
        torch.cuda.synchronize()
        times_q.append(a.elapsed_time(b))
        times_l.append(a.elapsed_time(c))
    qm = statistics.median(times_q[1:])
    out["delayed_16_steps"] = {"x_quantize_us_median_t_ge_1": qm * 1e3,
                               "x_quantize_GB_per_s": M * K * 3 / (qm * 1e-3) / 1e9,
                               "step0_quantize_us": times_q[0] * 1e3,
                               "linear_step_ms_median": statistics.median(times_l),
                               "gemm_tflops": 2 * M * N * K / ((statistics.median(times_l) - qm) * 1e-3) / 1e12}
    del xs_steps, wq, y, xq
    torch.cuda.empty_cache()
    # context: the same llama70b_prefill GEMM through cuBLASLt (torch._scaled_mm, per-row
    # scales, bf16 out) and through fp8_scaled_gemm, each 300 launches back to back
    try:
        from fp8_dynamic_scaled_b200 import inputs as _inp
        M, K, N = 4096, 8192, 28672
        xh, wh = _inp.llama70b_prefill(M, K, N)
        xq, xs, _ = fp8.empty_quant_outputs(M, K, fp8.FP8_SCALE_ROW)
        wq, wsc, _ = fp8.empty_quant_outputs(N, K, fp8.FP8_SCALE_ROW)
        fp8.fp8_quantize(to_dev_bf16(torch, xh), fp8.FP8_E4M3, fp8.FP8_SCALE_ROW, xq, xs)
        fp8.fp8_quantize(to_dev_bf16(torch, wh), fp8.FP8_E4M3, fp8.FP8_SCALE_ROW, wq, wsc)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        a8 = xq.view(torch.float8_e4m3fn)
        b8 = wq.view(torch.float8_e4m3fn).t()
        sa, sb = xs.view(M, 1), wsc.view(1, N)

        def run_ours():
            fp8.fp8_scaled_gemm(xq, xs, fp8.FP8_SCALE_ROW, fp8.FP8_E4M3, wq, wsc, fp8.FP8_SCALE_ROW, fp8.FP8_E4M3, y,
                                stream=stream)

        def run_cublas():
            torch._scaled_mm(a8, b8, scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)

        res = {}
        for name, fn in (("fp8_scaled_gemm", run_ours), ("cublaslt_scaled_mm", run_cublas)):
            with torch.cuda.stream(stream):
                for _ in range(5):
                    fn()
                torch.cuda.synchronize()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(300):
                    fn()
                b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / 300
            res[name] = {"us": ms * 1e3, "tflops": 2.0 * M * N * K / (ms * 1e-3) / 1e12}
        res["note"] = "library context only; same shapes, per-row scales, bf16 out, 300 back-to-back launches each"
        out["gemm_vs_cublaslt"] = res
    except Exception as ex:  # the comparison is context; a missing cuBLASLt FP8 path must not fail the bench
        out["gemm_vs_cublaslt"] = {"error": str(ex)[:200]}
    # epilogue options on the same layer: bias + output amax, FP8 output, and the unfused
    # equivalent of the FP8 output (bf16 Y, then a per-tensor quantize of Y)
    try:
        bias = torch.linspace(-1, 1, N, device="cuda").to(torch.bfloat16)
        amax = torch.zeros(1, device="cuda")
        s_y = torch.full((1,), 0.05, device="cuda")
        yq = torch.empty((M, N), dtype=torch.uint8, device="cuda")
        qy, sy, _ = fp8.empty_quant_outputs(M, N, fp8.FP8_SCALE_TENSOR)
        yws = fp8.workspace_for(0, M, 0, N, fp8.FP8_SCALE_TENSOR)
        R_, E4 = fp8.FP8_SCALE_ROW, fp8.FP8_E4M3
        variants = {
            "plain_bf16": lambda: fp8.fp8_scaled_gemm(xq, xs, R_, E4, wq, wsc, R_, E4, y, stream=stream),
            "bias_amax_bf16": lambda: fp8.fp8_scaled_gemm_ex(xq, xs, R_, E4, wq, wsc, R_, E4, y, bias=bias,
                                                             amax=amax, stream=stream),
            "bias_amax_fp8_only": lambda: fp8.fp8_scaled_gemm_ex(xq, xs, R_, E4, wq, wsc, R_, E4, None, bias=bias,
                                                                 amax=amax, yq=yq, yq_scale=s_y, stream=stream),
            "unfused_bias_bf16_then_quantize_y": lambda: (
                fp8.fp8_scaled_gemm_ex(xq, xs, R_, E4, wq, wsc, R_, E4, y, bias=bias, stream=stream),
                fp8.fp8_quantize(y, E4, fp8.FP8_SCALE_TENSOR, qy, sy, workspace=yws, stream=stream)),
        }
        # the variants are interleaved (5 rounds of 20 calls each) so that clock changes
        # under the power cap affect them alike; per variant the median round is reported
        per = {name: [] for name in variants}
        with torch.cuda.stream(stream):
            for fn in variants.values():
                fn()
        torch.cuda.synchronize()
        for _ in range(5):
            for name, fn in variants.items():
                with torch.cuda.stream(stream):
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    for _ in range(20):
                        fn()
                    b.record(stream)
                torch.cuda.synchronize()
                per[name].append(a.elapsed_time(b) / 20)
        res = {}
        for name, ts in per.items():
            ms = statistics.median(ts)
            res[name] = {"us": ms * 1e3, "gemm_tflops_equiv": 2.0 * M * N * K / (ms * 1e-3) / 1e12}
        res["note"] = "llama70b_prefill layer, per-row scales; 5 interleaved rounds of 20 calls, median round"
        out["epilogue_options"] = res
    except Exception as ex:
        out["epilogue_options"] = {"error": str(ex)[:200]}
    # decode-shaped calls of the same layer: M tokens against the 235 MB FP8 weight, which
    # no L2 holds, so every call streams W from HBM; the bound is W's bytes.  The GEMM loops
    # just before run the part at its power cap; an idle second lets the clocks come back
    # before these short calls, and the section records the clocks it saw.
    clk = ClockSampler(gpu_index)
    try:
        res = {}
        torch.cuda.synchronize()
        time.sleep(1.0)
        clk.__enter__()
        for Md in (1, 8, 16, 32, 64, 128, 256):
            yd = torch.empty((Md, N), dtype=torch.bfloat16, device="cuda")
            xd, xsd = xq[:Md], xs[:Md]

            def run_dec():
                fp8.fp8_scaled_gemm(xd, xsd, fp8.FP8_SCALE_ROW, fp8.FP8_E4M3, wq, wsc, fp8.FP8_SCALE_ROW,
                                    fp8.FP8_E4M3, yd, stream=stream)
            # per call: events around each of 50 calls, median; and the 50 calls back to
            # back between two events (that time also holds any gap between launches)
            ms, _ = time_kernel(torch, run_dec, 50, stream, warmup=5)
            with torch.cuda.stream(stream):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(50):
                    run_dec()
                b.record(stream)
            torch.cuda.synchronize()
            loop_ms = a.elapsed_time(b) / 50
            nbytes = N * K + Md * K + 4 * (Md + N) + 2 * Md * N
            res[f"M{Md}"] = {"us": ms * 1e3, "GB_per_s": nbytes / (ms * 1e-3) / 1e9,
                             "frac_of_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm,
                             "tflops": 2.0 * Md * N * K / (ms * 1e-3) / 1e12, "back_to_back_us": loop_ms * 1e3}
        res["note"] = ("N=28672, K=8192 per-row scales; bytes = W codes + X codes + scales + bf16 Y; us = median "
                       "of 50 calls each between two events; back_to_back_us = 50 calls between two events")
        # the whole decode layer: fp8_linear_forward (X quantize, then the GEMM launched as
        # its programmatic dependent, streaming W while X is quantised) against the same
        # two steps as separate calls; interleaved rounds of 50 calls, median round
        xh_all = inputs.llama70b_prefill(64, K, N, with_w=False)[0]
        for Md in (1, 16, 64):
            xd = to_dev_bf16(torch, xh_all[:Md])
            yd = torch.empty((Md, N), dtype=torch.bfloat16, device="cuda")
            lws = fp8.workspace_for(2, Md, N, K, fp8.FP8_SCALE_ROW)
            xq_d, xs_d, _ = fp8.empty_quant_outputs(Md, K, fp8.FP8_SCALE_ROW)
            qws = fp8.workspace_for(0, Md, 0, K, fp8.FP8_SCALE_ROW)
            fns = {
                "linear_forward": lambda: fp8.fp8_linear_forward(xd, fp8.FP8_E4M3, fp8.FP8_SCALE_ROW, wq, wsc,
                                                                 fp8.FP8_SCALE_ROW, fp8.FP8_E4M3, yd, lws,
                                                                 stream=stream),
                "quantize_then_gemm": lambda: (
                    fp8.fp8_quantize(xd, fp8.FP8_E4M3, fp8.FP8_SCALE_ROW, xq_d, xs_d, workspace=qws, stream=stream),
                    fp8.fp8_scaled_gemm(xq_d, xs_d, fp8.FP8_SCALE_ROW, fp8.FP8_E4M3, wq, wsc, fp8.FP8_SCALE_ROW,
                                        fp8.FP8_E4M3, yd, stream=stream)),
            }
            per = {k: [] for k in fns}
            with torch.cuda.stream(stream):
                for f in fns.values():
                    f()
            torch.cuda.synchronize()
            for _ in range(5):
                for k, f in fns.items():
                    with torch.cuda.stream(stream):
                        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        a.record(stream)
                        for _ in range(50):
                            f()
                        b.record(stream)
                    torch.cuda.synchronize()
                    per[k].append(a.elapsed_time(b) / 50 * 1e3)
            res[f"layer_M{Md}_us"] = {k: statistics.median(v) for k, v in per.items()}
        # weight-only FP8 (X stays bf16, W codes decoded on chip): the same layer; up to
        # 3 tokens on the CUDA-core matrix-vector kernel, above on the tensor-core one
        for Md in (1, 2, 3, 4, 16, 64):
            xd = to_dev_bf16(torch, xh_all[:Md])
            yd = torch.empty((Md, N), dtype=torch.bfloat16, device="cuda")
            med, _ = time_kernel(torch, lambda: fp8.fp8_weight_only_linear(xd, wq, wsc, fp8.FP8_SCALE_ROW, fp8.FP8_E4M3,
                                                                           yd, stream=stream), 50, stream)
            nbytes = N * K + 2 * Md * K + 4 * N + 2 * Md * N
            res[f"weight_only_M{Md}"] = {"us": med * 1e3, "GB_per_s": nbytes / (med * 1e-3) / 1e9,
                                         "frac_of_hbm": nbytes / (med * 1e-3) / 1e9 / hbm}
        clk.__exit__(None, None, None)
        res["clocks"] = clk.summary()
        out["decode_shapes"] = res
    except Exception as ex:
        clk.__exit__(None, None, None)
        out["decode_shapes"] = {"error": str(ex)[:200]}
    xq = wq = y = yq = qy = None      # release the layer's buffers
    torch.cuda.empty_cache()
    # small per-tensor linear (latency-bound)
    xh, wh = inputs.linear_small()
    x, w = to_dev_bf16(torch, xh), to_dev_bf16(torch, wh)
    wq, wsc, _ = fp8.empty_quant_outputs(256, 256, fp8.FP8_SCALE_TENSOR)
    fp8.fp8_quantize(w, fp8.FP8_E4M3, fp8.FP8_SCALE_TENSOR, wq, wsc,
                     workspace=fp8.workspace_for(0, 256, 0, 256, fp8.FP8_SCALE_TENSOR))
    y = torch.empty((128, 256), dtype=torch.bfloat16, device="cuda")
    lws = fp8.workspace_for(2, 128, 256, 256, fp8.FP8_SCALE_TENSOR)
    med, p95 = time_kernel(torch, lambda: fp8.fp8_linear_forward(x, fp8.FP8_E4M3, fp8.FP8_SCALE_TENSOR, wq, wsc,
                                                                 fp8.FP8_SCALE_TENSOR, fp8.FP8_E4M3, y, lws,
                                                                 stream=stream), 100, stream)
    # host cost of one call (argument checks, tensor maps, launches), no synchronisation
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        for _ in range(200):
            fp8.fp8_linear_forward(x, fp8.FP8_E4M3, fp8.FP8_SCALE_TENSOR, wq, wsc, fp8.FP8_SCALE_TENSOR, fp8.FP8_E4M3,
                                   y, lws, stream=stream)
    host_us = (time.perf_counter() - t0) / 200 * 1e6
    torch.cuda.synchronize()
    out["linear_small"] = {"us_median": med * 1e3, "us_p95": p95 * 1e3, "host_us_per_call": host_us}
    # the same call captured once in a CUDA graph (the calls allocate nothing and run on
    # the given stream) and replayed: the launch path without the per-call host work
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
            fp8.fp8_linear_forward(x, fp8.FP8_E4M3, fp8.FP8_SCALE_TENSOR, wq, wsc, fp8.FP8_SCALE_TENSOR,
                                   fp8.FP8_E4M3, y, lws, stream=stream)
        gmed, gp95 = time_kernel(torch, g.replay, 100, stream)
        out["linear_small"].update({"graph_replay_us_median": gmed * 1e3, "graph_replay_us_p95": gp95 * 1e3})
        del g
    except Exception as ex:
        out["linear_small"]["graph_replay_error"] = str(ex)[:200]
    return out


def config_summary(cfg):
    """The per-config headline numbers of the extras, flat (kept short so that a parser
    that keeps only top-level keys still sees them)."""
    out = {}
    def pick(key, *path):
        v = cfg
        for k in path:
            if not isinstance(v, dict) or k not in v:
                return
            v = v[k]
        out[key] = round(v, 4) if isinstance(v, float) else v
    pick("quant_sweep_e4m3_GB_s", "quant_sweep_e4m3", "GB_per_s")
    pick("quant_sweep_e4m3_frac_hbm", "quant_sweep_e4m3", "frac_of_hbm")
    pick("quant_sweep_e5m2_GB_s", "quant_sweep_e5m2", "GB_per_s")
    pick("quant_sweep_e5m2_frac_hbm", "quant_sweep_e5m2", "frac_of_hbm")
    pick("block_scaled_gemm_tflops", "block_scaled", "gemm_tflops")
    pick("block_scaled_gemm_frac_burst", "block_scaled", "gemm_frac_of_fp8_peak_burst")
    pick("block_scaled_x_quant_GB_s", "block_scaled", "x_quantize_GB_per_s")
    pick("mx_gemm_tflops", "mx", "gemm_tflops")
    pick("mx_gemm_frac_burst", "mx", "gemm_frac_of_fp8_peak_burst")
    pick("mx_x_quant_GB_s", "mx", "x_quantize_GB_per_s")
    pick("delayed_x_quant_GB_s", "delayed_16_steps", "x_quantize_GB_per_s")
    pick("decode_M16_frac_hbm", "decode_shapes", "M16", "frac_of_hbm")
    pick("decode_M64_frac_hbm", "decode_shapes", "M64", "frac_of_hbm")
    pick("weight_only_M16_us", "decode_shapes", "weight_only_M16", "us")
    pick("linear_small_us", "linear_small", "us_median")
    pick("linear_small_graph_us", "linear_small", "graph_replay_us_median")
    return out


# ---------------------------------------------------------------- CPU oracle (baseline / reference arm)
ORACLE_ROWS = 64           # the all-cores sample: X rows 0..63 of llama70b_prefill against all of W
ORACLE_ROWS_1T = 8         # the single-thread sample


def host_cores() -> int:
    """Cores this process may run on (the container's CPU set, else os.cpu_count())."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except (AttributeError, OSError):
        return max(1, os.cpu_count() or 1)


def _oracle_state(state={}):
    """W of llama70b_prefill quantised per channel by the oracle (once, untimed) and the
    first ORACLE_ROWS rows of X (the seeded workload's rows, generated directly)."""
    import oracle
    from fp8_dynamic_scaled_b200 import inputs
    if "qw" not in state:
        wl = WORKLOADS["llama70b_prefill"]
        x, w = inputs.llama70b_prefill(ORACLE_ROWS, wl["K"], wl["N"])
        with oracle.threads(host_cores()):
            qw, sw, _ = oracle.quantize(w, oracle.E4M3, oracle.ROW, dequant=False)
        state.update(x=x, qw=qw, sw=sw)
    return state


def oracle_sample_step(rows: int, threads: int):
    """The oracle's linear path on rows 0..rows-1 of the llama70b_prefill step: per-token
    quantisation of those X rows and the fp64 reference GEMM of those rows against all
    28,672 rows of W (K = 8192), on `threads` threads.  Returns (seconds, FLOPs)."""
    import oracle
    st = _oracle_state()
    x = np.ascontiguousarray(st["x"][:rows])
    with oracle.threads(threads):
        t0 = time.perf_counter()
        qx, sx, _ = oracle.quantize(x, oracle.E4M3, oracle.ROW, dequant=False)
        oracle.gemm_ref_slice(qx, sx, oracle.ROW, oracle.E4M3, st["qw"], st["sw"], oracle.ROW, oracle.E4M3, 0, rows)
        dt = time.perf_counter() - t0
    wl = WORKLOADS["llama70b_prefill"]
    return dt, 2.0 * rows * wl["N"] * wl["K"]


def oracle_sample_text(rows, threads):
    return (f"oracle (plain C, fp64 GEMM reference) on X rows 0..{rows - 1} of llama70b_prefill against all "
            f"28672 W rows (K=8192): per-token quantize of those rows + reference GEMM, {threads} thread(s); "
            f"W per-channel quantisation once, untimed; value = sample FLOPs / sample time")


def oracle_quantize_legs(cores: int):
    """The oracle's quantize step on the other workloads' activations, in GB/s of
    algorithmic bytes: all cores on the whole tensor, one thread on its first
    rows/16 rows (rate extrapolated to the whole tensor)."""
    import oracle
    from fp8_dynamic_scaled_b200 import inputs
    legs = {}
    cases = [("quant_sweep_e4m3_e5m2", lambda: inputs.quant_sweep(), oracle.TENSOR, True, 5),
             ("llama70b_prefill_x_per_token", lambda: inputs.llama70b_prefill(with_w=False)[0], oracle.ROW, False, 3),
             ("block_scaled_x_1x128", lambda: inputs.block_scaled(with_w=False)[0], oracle.BLOCK_1x128, False, 3),
             ("mx_x_mx32", lambda: inputs.mx_delayed(with_w=False)[0], oracle.MX32, False, 3)]
    for name, make, mode, deq, bpe in cases:
        x = make()
        fmts = (oracle.E4M3, oracle.E5M2) if name.startswith("quant_sweep") else (oracle.E4M3,)
        nbytes = x.size * bpe * len(fmts)
        res = {}
        for label, threads, sub in (("all_cores", cores, x), ("one_thread", 1, x[:max(1, x.shape[0] // 16)])):
            with oracle.threads(threads):
                t0 = time.perf_counter()
                for f in fmts:
                    oracle.quantize(np.ascontiguousarray(sub), f, mode, dequant=deq)
                dt = time.perf_counter() - t0
            frac = sub.shape[0] / x.shape[0]
            res[label] = {"GB_per_s": nbytes * frac / dt / 1e9, "threads": threads,
                          "rows_timed": int(sub.shape[0]), "extrapolated": frac < 1.0}
        legs[name] = res
        del x
    return legs


def run_reference(args):
    """The reference arm: the oracle (as it stands) on the host's cores, on a bounded
    sample of the same step (X rows 0..63 of llama70b_prefill against all of W)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cores = host_cores()
    for _ in range(args.warmup):
        oracle_sample_step(ORACLE_ROWS, cores)
    ts = []
    flops = 0.0
    for _ in range(args.steps):
        dt, flops = oracle_sample_step(ORACLE_ROWS, cores)
        ts.append(dt)
    ms = statistics.mean(ts) * 1e3
    value = flops / (ms * 1e-3) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "llama70b_prefill", "M": 4096, "N": 28672, "K": 8192,
                       "sample_rows": ORACLE_ROWS, "sample_cols": 28672},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": oracle_sample_text(ORACLE_ROWS, cores)},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def cpu_baseline_line():
    """cpu_baseline of the native line: the oracle's step sample on all cores (the
    value) and on one thread, plus the quantize legs of the other workloads."""
    cores = host_cores()
    oracle_sample_step(ORACLE_ROWS_1T, cores)                  # warm-up (W codes, page-in)
    ts = [oracle_sample_step(ORACLE_ROWS, cores)[0] for _ in range(2)]
    fl = oracle_sample_step(ORACLE_ROWS, cores)[1]
    dt = min(ts)
    dt1, fl1 = oracle_sample_step(ORACLE_ROWS_1T, 1)
    full_flops = 2.0 * 4096 * 28672 * 8192
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": oracle_sample_text(ORACLE_ROWS, cores) + "; best of 2",
            "one_thread": {"value": fl1 / dt1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                           "sample": oracle_sample_text(ORACLE_ROWS_1T, 1)},
            "full_step_s_extrapolated": {"all_cores": dt * full_flops / fl, "one_thread": dt1 * full_flops / fl1,
                                         "note": "the sample's time scaled linearly to the 4096 rows of the step"},
            "host_cpu_count": os.cpu_count(),
            "quantize_legs": oracle_quantize_legs(cores)}


def run_quant_sweep(args, torch, fp8, stream, barrier, dist, world, rank, gpu_index, peaks, peak_src):
    """Workload ``quant_sweep``: a 64 Mi-element bf16 tensor (log-uniform magnitudes over
    [1e-6, 1e4], random signs, 1e-4 outliers at +-1e5); one step = per-tensor current
    scaling to E4M3 and to E5M2, each emitting codes + fp32 scale + dequantised bf16."""
    from fp8_dynamic_scaled_b200 import inputs
    xh = rank_batch(inputs.quant_sweep(), rank)
    x = to_dev_bf16(torch, xh)
    rows, cols = x.shape
    T = fp8.FP8_SCALE_TENSOR
    outs = {f: fp8.empty_quant_outputs(rows, cols, T, dequant=True) for f in (fp8.FP8_E4M3, fp8.FP8_E5M2)}
    ws = fp8.workspace_for(0, rows, 0, cols, T)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    per_fmt = rows * cols * (2 + 1 + 2) + 4

    def step(evs=None):
        for i, f in enumerate((fp8.FP8_E4M3, fp8.FP8_E5M2)):
            q, sc, d = outs[f]
            if evs:
                evs[i][0].record(stream)
            fp8.fp8_quantize(x, f, T, q, sc, dequant=d, dev_status=status, workspace=ws, stream=stream)
            if evs:
                evs[i][1].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(2)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if barrier:
        barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_index) as clk:
        with torch.cuda.stream(stream):
            start.record(stream)
            for i in range(args.steps):
                step(evs[i])
            end.record(stream)
        torch.cuda.synchronize()
    if barrier:
        barrier()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}")
    total_ms = max_over_ranks(start.elapsed_time(end), dist, "cuda")
    ms = total_ms / args.steps
    value = whole_job_rate(2 * per_fmt, world, ms) / 1e9
    k_ms = statistics.mean(e[i][0].elapsed_time(e[i][1]) for e in evs for i in range(2))
    achieved = per_fmt / (k_ms * 1e-3) / 1e9
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16->e4m3/e5m2", "data": "synthetic",
            "config": {"workload": "quant_sweep", "elements": rows * cols, "scaling": "per-tensor current",
                       "formats": ["e4m3", "e5m2"], "outputs": "codes + fp32 scale + bf16 dequant",
                       "l2": "inputs larger than L2 (each call reads 128 MB, writes 192 MB)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"],
                         "traffic": profiled_traffic("quant_tensor_quant_sweep"),
                         "kernel": "rq_persist_kernel (one fp8_quantize call: a single cooperative launch)",
                         "peak_source": f"{peak_src} hbm_gbs", "call_us_avg": k_ms * 1e3},
            "clocks": clk.summary(), "gpu_launches": args.steps * 4}
    if rank == 0:
        q, sc, d = outs[fp8.FP8_E4M3]
        x_pin = torch.from_numpy(np.ascontiguousarray(xh).view(np.int16)).view(torch.bfloat16).pin_memory()
        pins = {f: (torch.empty((rows, cols), dtype=torch.uint8).pin_memory(),
                    torch.empty((rows, cols), dtype=torch.bfloat16).pin_memory()) for f in outs}
        xd = torch.empty_like(x)

        def e2e_step():
            xd.copy_(x_pin, non_blocking=True)
            for f in (fp8.FP8_E4M3, fp8.FP8_E5M2):
                q, sc, d = outs[f]
                fp8.fp8_quantize(xd, f, T, q, sc, dequant=d, workspace=ws, stream=stream)
                pins[f][0].copy_(q, non_blocking=True)
                pins[f][1].copy_(d, non_blocking=True)

        n = max(3, min(args.steps, 10))
        with torch.cuda.stream(stream):
            e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for _ in range(n):
                e2e_step()
            b.record(stream)
        torch.cuda.synchronize()
        e_ms = a.elapsed_time(b) / n
        line["e2e"] = {"value": world * 2 * per_fmt / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
                       "h2d_bytes_per_step": rows * cols * 2, "d2h_bytes_per_step": 2 * rows * cols * 3,
                       "ms_per_step": e_ms, "api": "fp8_quantize with pinned host X in / codes+dequant out"}
        print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama70b_prefill", choices=sorted(WORKLOADS) + ["quant_sweep"])
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    args.warmup = max(args.warmup, 3)

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    from fp8_dynamic_scaled_b200 import binding as fp8
    if fp8.fp8_device_check() != fp8.FP8_OK:
        raise SystemExit("not an sm_100 device")
    peaks, peak_src = load_peaks()
    stream = torch.cuda.Stream()
    barrier = (lambda: dist.barrier()) if dist else None

    gpu_index = local_rank
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        gpu_index = int(vis.split(",")[local_rank])
    if args.workload == "quant_sweep":
        return run_quant_sweep(args, torch, fp8, stream, barrier, dist, world, rank, gpu_index, peaks, peak_src)
    wl = make_workload(torch, fp8, args.workload, rank)
    M, K, N = wl["M"], wl["K"], wl["N"]
    with ClockSampler(gpu_index) as clk:
        total_ms, q_ms, g_ms, _ = time_linear_steps(torch, fp8, wl, args.steps, args.warmup, stream, barrier)
    clocks = clk.summary()
    total_ms = max_over_ranks(total_ms, dist, "cuda")
    ms_per_step = total_ms / args.steps
    flops = 2.0 * M * N * K
    value = whole_job_rate(flops, world, ms_per_step) / 1e12
    g_avg = statistics.mean(g_ms)
    q_avg = statistics.mean(q_ms)
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * FP8_OVER_BF16
    sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]) * FP8_OVER_BF16
    use_sustained, capped = use_sustained_peak(total_ms, clocks)
    fp8_peak = sustained if use_sustained else burst
    gemm_tflops = flops / (g_avg * 1e-3) / 1e12
    variant = {1: "ROWSCALE", 2: "BLOCK", 4: "MX"}[wl["x_mode"]]
    traffic = profiled_traffic(f"gemm_{variant.lower()}_{args.workload}")
    xbytes = M * K * 3 + {1: 4 * M, 2: 4 * M * (-(-K // 128)), 4: M * (K // 32)}[wl["x_mode"]]
    qkernel = {1: "rq_row_kernel", 2: "rq_block_kernel<B128>", 4: "rq_block_kernel<MX>"}[wl["x_mode"]]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": args.workload, "M": M, "N": N, "K": K,
                   "x_scaling": {1: "per-token", 2: "1x128 blocks", 4: "MX32"}[wl["x_mode"]],
                   "w_scaling": {1: "per-channel", 3: "128x128 blocks", 4: "MX32"}[wl["w_mode"]],
                   "fp8": "e4m3", "out": "bf16",
                   "l2": f"inputs larger than L2 (each step reads {2 * M * K / 1e6:.0f} MB X + "
                         f"{N * K / 1e6:.0f} MB W codes, writes {2 * M * N / 1e6:.0f} MB Y)"},
        "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": gemm_tflops / fp8_peak, "traffic": traffic,
                     "peak_kind": "sustained" if use_sustained else "burst",
                     "frac_of_burst": gemm_tflops / burst, "frac_of_sustained": gemm_tflops / sustained,
                     "timed_region_ms": total_ms, "power_cap_seen": capped,
                     "kernel": "fp8_gemm_pair_kernel" if variant == "ROWSCALE" and M >= 256 else f"fp8_gemm_kernel<{variant}>",
                     "peak_source": f"{peak_src} bf16 {'sustained' if use_sustained else 'burst'} x "
                                    f"{FP8_OVER_BF16} (fp8/bf16 nominal ratio); sustained only for a timed region "
                                    f">= 1 s that saw sw_power_cap",
                     "gemm_us_avg": g_avg * 1e3},
    }
    if variant == "ROWSCALE" and M <= 64:
        # few tokens: the GEMM is bound by streaming W (and X, scales, Y) from HBM
        gbytes = N * K + M * K + 4 * (M + N) + 2 * M * N
        line["roofline"] = {"bound": "hbm", "achieved": gbytes / (g_avg * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                            "unit": "GB/s", "frac": gbytes / (g_avg * 1e-3) / 1e9 / peaks["hbm_gbs"],
                            "traffic": profiled_traffic(f"gemm_decode_{args.workload}"), "kernel": "fp8_decode_kernel",
                            "peak_source": f"{peak_src} hbm_gbs", "gemm_us_avg": g_avg * 1e3,
                            "algorithmic_bytes": gbytes, "gemm_tflops": gemm_tflops}
    line.update({
        "quantize": {"kernel": qkernel, "us_avg": q_avg * 1e3, "algorithmic_bytes": xbytes,
                     "GB_per_s": xbytes / (q_avg * 1e-3) / 1e9,
                     "frac_of_hbm": xbytes / (q_avg * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "share_of_gemm_time": q_avg / g_avg},
        "clocks": clocks,
        "gpu_launches": args.steps * (quantize_launches(wl["x_mode"]) + 1),
    })
    if rank == 0:
        e2e_ms, h2d, d2h = time_e2e(torch, fp8, wl, max(3, min(args.steps, 20)), 2, stream)
        line["e2e"] = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                       "api": "fp8_linear_forward with pinned host X in / Y out, copies on their own streams "
                              "(two buffers; uploads, compute and downloads of neighbouring steps overlap)"}
        del wl
        torch.cuda.empty_cache()
        if world == 1 and not args.no_extras:
            line["configs"] = extras(torch, fp8, stream, peaks, gpu_index)
            line["summary"] = config_summary(line["configs"])
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_line()
        print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
