"""Benchmark of the 4-bit weight-only quantized product hot path on B200.

One *step* runs every hot-path operation once on synthetic Llama/Qwen-shaped
layers (seeded, weights N(0, 0.02) quantized on the GPU, activations N(0, 1)
with outlier channels):

  nf4_dequant   NF4 -> bf16, W [28672 x 8192]                      (HBM-bound)
  gemv_int4     decode GEMV, M = 16, W [11008 x 4096], INT4 g128    (HBM-bound)
  gemv_nf4      decode GEMV, M = 16, W [11008 x 4096], NF4 b64      (HBM-bound)
  gemm          prefill GEMM, M = 8192, W [14336 x 4096], INT4 g128 (tensor-bound)
  msd_m16       MSD GEMM, C = 2, M = 16, W [25600 x 5120], g128     (HBM-bound)
  msd_m1024     MSD GEMM, C = 2, M = 1024, W [25600 x 5120], g128   (tensor-bound)

Metric: "% of B200 roofline" of the whole step, work-weighted: for every op
its roofline time max(algorithmic bytes / HBM peak, algorithmic ops / tensor
peak) is summed, and divided by the measured step time. The tensor peak is the
measured bf16 burst figure, or the sustained one if this run's own clock
record shows the power cap (or clocks well below maximum); int8 is twice
bf16. With N GPUs each rank runs its own replica (no data-path collective)
and the value is the sum over ranks (weak scaling; 100 per GPU is the
ceiling).

Timing: W untimed warm-up steps, then exactly K steps between a barrier +
synchronize on both sides, CUDA events on the launching stream, max over
ranks. L2: every op's weights were last touched one step earlier and the
600 MB NF4 dequantization stream (> 4x the 126 MB L2) runs in between (each op
has its own weights), so every op's weights start L2-cold. `--impl reference`
times the CPU oracle on a bounded sample of the same step instead (rank 0
only).

After the step (outside its value): the dequantize-then-cuBLAS comparator,
the salient-channel correction rows, and `per_config`, the throughput and
roofline fraction of every workload of the five configurations, each
graph-timed over rotating weight copies larger than 4x L2 with its own clock
median.
"""

import argparse
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-GEMM GB/s (decode) & TFLOP/s (prefill) as % of B200 roofline"
UNIT = "% of one B200 roofline (work-weighted over the step, summed over GPUs)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

GEMV_SHAPE = (11008, 4096)
GEMM_SHAPE = (8192, 14336, 4096)
MSD_SHAPE = (25600, 5120)
NF4_SHAPE = (28672, 8192)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def tensor_peak(peaks, clocks):
    """The bf16 tensor peak (TFLOP/s) that matches the clocks recorded while
    the timed work ran: the burst figure (measured for a kernel timed alone at
    full clock) unless the power cap was active or the SM clock sat well below
    its maximum, in which case the sustained figure (measured back to back for
    seconds, under the cap). Returns (TFLOP/s, "burst" | "sustained")."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = "sw_power_cap" in clocks.get("reasons", [])
    if capped or (mhz and mx and mhz < 0.9 * mx):
        return peaks["bf16_tflops_sustained"], "sustained"
    return peaks["bf16_tflops"], "burst"


def op_table(peaks, tf16_tflops):
    """Algorithmic bytes and ops of each op of the step, with its roofline time.

    Bytes: packed weights (0.5 B/weight) + scales/zeros or absmax + activations
    read + outputs written; ops: 2*M*N*K multiply-adds (x2 components for MSD).
    tf16_tflops is the bf16 tensor peak chosen by tensor_peak(); the int8 peak
    is twice it (dense int8 runs at twice the bf16 rate on B200)."""
    bw = peaks["hbm_gbs"] * 1e9
    tf16 = tf16_tflops * 1e12
    ti8 = 2.0 * tf16
    n, k = NF4_SHAPE
    gn, gk = GEMV_SHAPE
    m, pn, pk = GEMM_SHAPE
    sn, sk = MSD_SHAPE
    ops = {
        "nf4_dequant": dict(bytes=n * k * (0.5 + 4 / 64 + 2), flops=0, peak_flops=tf16, bound="hbm"),
        "gemv_int4": dict(bytes=gn * gk * (0.5 + 4 / 128) + 2 * 16 * gk + 2 * 16 * gn,
                          flops=2 * 16 * gn * gk, peak_flops=tf16, bound="hbm"),
        "gemv_nf4": dict(bytes=gn * gk * (0.5 + 4 / 64) + 2 * 16 * gk + 2 * 16 * gn,
                         flops=2 * 16 * gn * gk, peak_flops=tf16, bound="hbm"),
        "gemm": dict(bytes=pn * pk * (0.5 + 4 / 128) + 2 * m * pk + 2 * m * pn,
                     flops=2 * m * pn * pk, peak_flops=tf16, bound="tensor"),
        "msd_m16": dict(bytes=sn * sk * (0.5 + 4 / 128) + 2 * 16 * sk + 2 * 16 * sn,
                        flops=2 * 2 * 16 * sn * sk, peak_flops=ti8, bound="hbm"),
        "msd_m1024": dict(bytes=sn * sk * (0.5 + 4 / 128) + 2 * 1024 * sk + 2 * 1024 * sn,
                          flops=2 * 2 * 1024 * sn * sk, peak_flops=ti8, bound="tensor"),
    }
    for v in ops.values():
        v["t_roof"] = max(v["bytes"] / bw, v["flops"] / v["peak_flops"] if v["flops"] else 0.0)
    return ops


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every `period` s,
    with wall-clock stamps, so that any window of the run (one case) can be
    summarised on its own."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle"}

    def __init__(self, index, period=0.05):
        self.samples, self.max_mhz, self.period = [], None, period  # (t, mhz, reasons)
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                names = {name for bit, name in self.REASONS.items()
                         if mask & bit and name != "gpu_idle"}
                self.samples.append((time.time(), mhz, names))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self, t0=None, t1=None):
        sel = [(m, r) for t, m, r in self.samples
               if (t0 is None or t >= t0) and (t1 is None or t <= t1)]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                    "reasons": ["unavailable" if not self._ok else "no sample in window"]}
        reasons = set()
        for _, r in sel:
            reasons |= r
        return {"sm_mhz": statistics.median(m for m, _ in sel), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(sel)}


# ---------------------------------------------------------------------------
# the GPU step
# ---------------------------------------------------------------------------

class Step:
    """Device-resident inputs, outputs and workspaces of one hot-path step."""

    def __init__(self, wq, device, seed=0):
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        self.wq = wq
        F = wq.WQ_FMT_INT4_ASYM

        def normal(*shape, std=1.0):
            return torch.randn(*shape, generator=g, device=device) * std

        def acts(m, k, frac, scale):
            x = normal(m, k)
            idx = torch.randperm(k, generator=g, device=device)[:max(1, round(frac * k))]
            x[:, idx] *= scale
            return x.to(torch.bfloat16)

        n, k = NF4_SHAPE
        w = normal(n, k, std=0.02)
        self.nf4_codes, self.nf4_absmax, _ = wq.wq_quantize_pack(wq.WQ_FMT_NF4, w, 64)
        del w
        self.nf4_out = torch.empty(n * k, dtype=torch.bfloat16, device=device)

        gn, gk = GEMV_SHAPE
        w = normal(gn, gk, std=0.02)
        self.gi = wq.wq_quantize_pack(F, w, 128)
        self.gn = wq.wq_quantize_pack(wq.WQ_FMT_NF4, w, 64)
        del w
        self.gx = acts(16, gk, 0.01, 20.0)
        self.gy_i = torch.empty(16, gn, dtype=torch.bfloat16, device=device)
        self.gy_n = torch.empty(16, gn, dtype=torch.bfloat16, device=device)

        m, pn, pk = GEMM_SHAPE
        w = normal(pn, pk, std=0.02)
        self.pw = wq.wq_quantize_pack(F, w, 128)
        del w
        self.px = normal(m, pk).to(torch.bfloat16)
        self.py = torch.empty(m, pn, dtype=torch.bfloat16, device=device)
        self.pws = wq.gemm_workspace(m, pn, pk, 128, device)

        sn, sk = MSD_SHAPE
        w = normal(sn, sk, std=0.02)
        self.sw = wq.wq_quantize_pack(F, w, 128)
        # the decode MSD op has its own copy of the layer: the prefill MSD op's
        # weights are read only the two GEMVs (~50 MB, under L2) before it
        self.sw16 = wq.wq_quantize_pack(F, w, 128)
        del w
        self.sx16 = acts(16, sk, 0.005, 50.0)
        self.sx1024 = acts(1024, sk, 0.005, 50.0)
        self.sy16 = torch.empty(16, sn, dtype=torch.bfloat16, device=device)
        self.sy1024 = torch.empty(1024, sn, dtype=torch.bfloat16, device=device)
        self.sws16 = wq.msd_workspace(16, sn, sk, 128, 2, device)
        self.sws1024 = wq.msd_workspace(1024, sn, sk, 128, 2, device)
        torch.cuda.synchronize()

    LAUNCHES_PER_STEP = 9  # nf4 1, gemv 2, gemm 2 (x->fp16 + GEMM), msd 2 x 2 (decompose + GEMM)

    def ops(self):
        wq = self.wq
        n, k = NF4_SHAPE
        gn, _ = GEMV_SHAPE
        _, pn, _ = GEMM_SHAPE
        sn, _ = MSD_SHAPE
        # Decode ops first: right after the 600 MB NF4 stream the GPU is still
        # writing that stream's dirty L2 lines back to HBM, which the
        # compute-bound GEMM absorbs and a 24 MB weight read does not. Every
        # op's inputs are still last touched a step earlier, with the NF4
        # stream in between.
        return [
            ("gemv_int4", lambda: wq.wq_w4a16_gemv(self.gx, gn, wq.WQ_FMT_INT4_ASYM, 128,
                                                   *self.gi, out=self.gy_i)),
            ("gemv_nf4", lambda: wq.wq_w4a16_gemv(self.gx, gn, wq.WQ_FMT_NF4, 64, *self.gn,
                                                  out=self.gy_n)),
            ("msd_m16", lambda: wq.wq_msd_gemm(self.sx16, sn, 2, 128, *self.sw16,
                                               workspace=self.sws16, out=self.sy16)),
            ("nf4_dequant", lambda: wq.wq_nf4_dequant(self.nf4_codes, self.nf4_absmax, n * k,
                                                      out=self.nf4_out)),
            ("gemm", lambda: wq.wq_w4a16_gemm(self.px, pn, wq.WQ_FMT_INT4_ASYM, 128, *self.pw,
                                              workspace=self.pws, out=self.py)),
            ("msd_m1024", lambda: wq.wq_msd_gemm(self.sx1024, sn, 2, 128, *self.sw,
                                                 workspace=self.sws1024, out=self.sy1024)),
        ]


def captured_traffic(op):
    """DRAM bytes (read + write) per launch of `op` from the committed ncu
    summary, or None when that kernel's source changed since the capture."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(prof):
        return None
    with open(prof) as f:
        entry = json.load(f).get(op)
    if not entry:
        return None
    with open(os.path.join(ROOT, entry["source"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != entry["source_sha"]:
            return None
    return entry["bytes_per_launch"]


def job_value(table, ms_per_step, world):
    """Whole-job value: 100 x (roofline time of one GPU's step) / (the slowest
    rank's step time) x ranks. Each replica runs the full step (weak
    scaling), so the work grows with the number of GPUs."""
    roof_ms = sum(v["t_roof"] for v in table.values()) * 1e3
    return 100.0 * roof_ms / ms_per_step * world


def dequant_then_cublas(wq, step, fused_ms, warmup):
    """The dequantize-then-bf16-GEMM baseline on the step's GEMM workload: the
    library's INT4 dequantization to a bf16 [N, K] weight, then torch.matmul
    (cuBLAS). Timed after the step's timed region, outside ms_per_step."""
    m, n, k = GEMM_SHAPE
    qw, sc, zr = step.pw
    wd = torch.empty(n, k, dtype=torch.bfloat16, device=step.px.device)
    y = torch.empty(m, n, dtype=torch.bfloat16, device=step.px.device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    reps = 5
    t_deq = t_mm = 0.0
    for i in range(max(warmup, 1) + reps):
        ev[0].record()
        wq.wq_int4_dequant(qw, sc, zr, n, k, 128, out=wd)
        ev[1].record()
        torch.matmul(step.px, wd.t(), out=y)
        ev[2].record()
        torch.cuda.synchronize()
        if i >= max(warmup, 1):
            t_deq += ev[0].elapsed_time(ev[1]) / reps
            t_mm += ev[1].elapsed_time(ev[2]) / reps
    # the same comparison at smaller prefill sizes (the first rows of the step's
    # x): the dequantization is a fixed cost per call, so its share grows as M
    # shrinks
    sweep = []
    for ms in (512, 2048, 4096):
        xs = step.px[:ms]
        ys = torch.empty(ms, n, dtype=torch.bfloat16, device=step.px.device)
        ws = wq.gemm_workspace(ms, n, k, 128, step.px.device)
        t_f = t_c = 0.0
        for i in range(max(warmup, 1) + reps):
            ev[0].record()
            wq.wq_w4a16_gemm(xs, n, wq.WQ_FMT_INT4_ASYM, 128, qw, sc, zr, workspace=ws, out=ys)
            ev[1].record()
            wq.wq_int4_dequant(qw, sc, zr, n, k, 128, out=wd)
            torch.matmul(xs, wd.t(), out=ys)
            ev[2].record()
            torch.cuda.synchronize()
            if i >= max(warmup, 1):
                t_f += ev[0].elapsed_time(ev[1]) / reps
                t_c += ev[1].elapsed_time(ev[2]) / reps
        sweep.append({"m": ms, "fused_ms": round(t_f, 4), "dequant_then_cublas_ms": round(t_c, 4),
                      "fused_speedup": round(t_c / t_f, 3)})
        del ys, ws
    del wd, y
    flops = 2.0 * m * n * k
    return {"workload": "gemm int4-g128 %dx%dx%d" % (m, n, k),
            "sweep_smaller_m": sweep,
            "dequant_then_cublas_ms": round(t_deq + t_mm, 4), "dequant_ms": round(t_deq, 4),
            "cublas_bf16_ms": round(t_mm, 4),
            "dequant_then_cublas_tflops": round(flops / ((t_deq + t_mm) * 1e-3) / 1e12, 1),
            "fused_gemm_ms": round(fused_ms, 4),
            "fused_tflops": round(flops / (fused_ms * 1e-3) / 1e12, 1),
            "fused_speedup": round((t_deq + t_mm) / fused_ms, 3)}


DECDEC_SHAPE = (11008, 4096)   # decode layer (N, K), INT4 g128
DECDEC_K = 64                   # salient channels corrected per step (1.6 % of K)


def _graph_us(fns, reps):
    """Median over 5 replays of a CUDA graph of `reps` launches cycling over
    fns, in microseconds per launch (device time, CUDA events)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for f in fns:
            f()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(reps):
            fns[i % len(fns)]()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ts = []
    for _ in range(5):
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) * 1e3 / reps)
    del g
    return statistics.median(ts)


def measure_decdec(wq, peaks, device, with_oracle):
    """Salient-channel residual correction ("DecDEC: A Systems Approach to
    Advancing Low-Bit LLM Quantization", Abstract), a widening beyond the step:
    the decode GEMV at 11008x4096 INT4 g128 plain and with the residuals of the
    64 most salient channels added, graph-timed over 8 rotating copies of the
    weights and residuals (their touched bytes exceed L2). Timed outside the
    step and not part of its value."""
    n, k = DECDEC_SHAPE
    copies = 8
    sets = []
    for c in range(copies):
        w = torch.randn(n, k, device=device, generator=torch.Generator(device=device).manual_seed(
            900 + c)) * 0.02
        qw, sc, zr = wq.wq_quantize_pack(wq.WQ_FMT_INT4_ASYM, w, 128)
        sets.append((w, qw, sc, zr, torch.empty(k, n, dtype=torch.float16, device=device)))
    res_us = _graph_us([lambda t=t: wq.wq_residual(wq.WQ_FMT_INT4_ASYM, t[0], 128, t[1], t[2],
                                                   t[3], out=t[4]) for t in sets], 16)
    res_bytes = n * k * (4 + 0.5 + 2) + n * (k // 128) * 4
    out = {"workload": "decode gemv int4-g128 %dx%d, residuals of %d salient channels"
                       % (n, k, DECDEC_K),
           "residual_us": round(res_us, 2),
           "residual_gbs": round(res_bytes / (res_us * 1e-6) / 1e9, 1),
           "residual_frac": round(res_bytes / (res_us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)}
    for m in (1, 16):
        x = (torch.randn(m, k, device=device, generator=torch.Generator(device=device).manual_seed(
            950 + m))).to(torch.bfloat16)
        x[:, ::64] *= 20.0  # outlier channels, 1.6 % of K
        idx = torch.empty(DECDEC_K, dtype=torch.int32, device=device)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
        plain = _graph_us([lambda t=t: wq.wq_w4a16_gemv(x, n, wq.WQ_FMT_INT4_ASYM, 128, t[1], t[2],
                                                        t[3], out=y) for t in sets], 32)
        sel = _graph_us([lambda: wq.wq_select_salient(x, DECDEC_K, out=idx)], 32)
        corr = _graph_us([lambda t=t: wq.wq_w4a16_gemv_corrected(
            x, n, wq.WQ_FMT_INT4_ASYM, 128, t[1], t[2], t[3], t[4], idx, out=y)
            for t in sets], 32)
        step_us = _graph_us([lambda t=t: wq.wq_w4a16_gemv_salient(
            x, n, wq.WQ_FMT_INT4_ASYM, 128, t[1], t[2], t[3], t[4], DECDEC_K, idx=idx, out=y)
            for t in sets], 32)
        gemv_bytes = n * k * 0.5 + n * (k // 128) * 4 + 2 * m * k + 2 * m * n
        corr_bytes = DECDEC_K * n * 2
        out["m%d" % m] = {
            "gemv_us": round(plain, 2), "select_us": round(sel, 2),
            "corrected_gemv_us": round(corr, 2),
            "overhead_pct": round(100.0 * (corr + sel - plain) / plain, 1),
            "salient_step_us": round(step_us, 2),
            "salient_step_overhead_pct": round(100.0 * (step_us - plain) / plain, 1),
            "correction_bytes": corr_bytes,
            "corrected_gemv_gbs": round((gemv_bytes + corr_bytes) / (corr * 1e-6) / 1e9, 1)}
    if with_oracle:
        out["cpu_baseline"] = decdec_cpu_baseline()
    del sets
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
# per-config throughput: every workload of the five configurations
# ---------------------------------------------------------------------------

L2_BYTES = 126 * 2 ** 20


def _copies_for(nbytes):
    """Weight copies whose total exceeds 4x L2 (at least 1, at most 1024)."""
    return int(max(1, min(1024, -(-4 * L2_BYTES // max(1, int(nbytes))))))


def _timed_launches(fns, sampler, min_ms=60.0):
    """Mean device time (us) of one call of fns[i] in a stream of back-to-back
    calls: the calls are captured as one CUDA graph, cycling over fns (each
    call on its own copy of the weights, so a copy is read again only after
    > 4x L2 of other copies), and the graph is replayed between two CUDA
    events until at least min_ms of device time is averaged; time / calls.
    (Events around every call inside the graph would add ~4 us each, measured
    on B200, which swamps decode-size kernels.) Returns (us, clocks of the
    replays)."""
    n = len(fns)
    reps = max(n, 16)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for f in fns[:2]:
            f()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(reps):
            fns[i % n]()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    total, cnt = 0.0, 0
    t0 = time.time()
    while True:
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        total += a.elapsed_time(b)
        cnt += reps
        if total >= min_ms and cnt >= 2 * reps:
            break
    t1 = time.time()
    del g
    return 1e3 * total / cnt, sampler.summary(t0, t1)


def measure_per_config(wq, peaks, device):
    """Absolute throughput and roofline fraction of every workload of the
    five configurations (timed after the step, not part of its value):

      1  decode GEMV, INT4 g64, M = 1, 1024 x 1024
      2  NF4 dequantization, 28672 x 8192, 8192 x 8192, 5120 x 25600
      3  decode GEMV, M = 1, 4, 8, 16 x (4096 x 4096, 11008 x 4096,
         4096 x 11008), INT4 g128 and NF4 b64, 1 % outlier channels x 20
      4  prefill fused GEMM, M = 512, 2048, 8192 x (4096 x 4096,
         14336 x 4096, 4096 x 14336), INT4 g128, beside dequantize-then-cuBLAS
      5  MSD GEMM, C = 2, M = 1, 16, 128, 1024 x (5120 x 5120, 25600 x 5120,
         5120 x 25600), per-channel and g128, 0.5 % outlier channels x 50;
         at M = 128 and 1024 (g128) beside the fused GEMM on the same layer,
         and the relative L2 errors of MSD and of the bf16
         dequantize-then-cuBLAS product against the exact product
      MX  the MX path of MSD on the same shapes at M = 1 and 16: MXFP4
         weights with two MXFP4 activation passes, and one MXFP8 pass
      NF4 MSD with NF4 weights (integer codebook digits), same shapes, M = 1
         and 16
      KV  MSD decode attention over an INT4 KV cache, C = 2, Qwen3-32B heads
         (Hq = 64, Hkv = 8, D = 128), B x L = 32 x 8192 and 8 x 32768,
         beside torch's scaled-dot-product attention on a bf16 cache (bytes:
         K and V codes with their fp16 scales and zeros, q and out)

    Each workload is graph-timed as a stream of back-to-back calls over
    rotating copies of its weights (> 4x L2 in total), with its own SM clock
    median. Bytes and ops are the
    algorithmic ones: packed weights, scales/zeros or absmax, activations
    read and outputs written; 2MNK flops (x C for MSD). Peaks: measured HBM
    copy; bf16 and int8 (2x bf16) tensor peaks, burst or sustained by each
    case's own clocks."""
    g = torch.Generator(device=device)
    g.manual_seed(1234)
    F, NF = wq.WQ_FMT_INT4_ASYM, wq.WQ_FMT_NF4
    bw = peaks["hbm_gbs"] * 1e9
    out = {"config1_gemv_tiny": [], "config2_nf4_dequant": [], "config3_gemv": [],
           "config4_gemm": [], "config5_msd": [], "msd_vs_fused_gemm": [], "msd_accuracy": [],
           "mx_msd_decode": [], "nf4_msd_decode": [], "kv_msd_decode_attention": []}

    def normal(*shape, std=1.0):
        return torch.randn(*shape, generator=g, device=device) * std

    def acts(m, k, frac, scale):
        x = normal(m, k)
        if frac:
            idx = torch.randperm(k, generator=g, device=device)[:max(1, round(frac * k))]
            x[:, idx] *= scale
        return x.to(torch.bfloat16)

    def packed_bytes(fmt, n, k, group):
        return n * k // 2 + (n * k // 64 * 4 if fmt == NF else n * (k // group) * 4)

    def weight_copies(fmt, n, k, group):
        one = wq.wq_quantize_pack(fmt, normal(n, k, std=0.02), group)
        r = _copies_for(packed_bytes(fmt, n, k, group))
        return [one] + [tuple(t.clone() if t is not None else None for t in one)
                        for _ in range(r - 1)]

    def entry(name, us, clk, nbytes, flops, int8=False, extra=None, fp8=False):
        tf16_kind = tensor_peak(peaks, clk)
        tpk = (2.0 if (int8 or fp8) else 1.0) * tf16_kind[0] * 1e12
        t_roof = max(nbytes / bw, flops / tpk if flops else 0.0)
        e = {"case": name, "us": round(us, 2), "gbs": round(nbytes / (us * 1e-6) / 1e9, 1),
             "tflops": round(flops / (us * 1e-6) / 1e12, 1),
             "bound": "hbm" if nbytes / bw >= (flops / tpk if flops else 0.0) else "tensor",
             "roofline_frac": round(t_roof / (us * 1e-6), 4),
             "peak": "hbm %.0f GB/s, %s %s %.0f TFLOP/s" % (
                 peaks["hbm_gbs"], tf16_kind[1], "fp8" if fp8 else ("int8" if int8 else "bf16"),
                 tpk / 1e12),
             "sm_mhz": clk.get("sm_mhz"), "clock_reasons": clk.get("reasons")}
        if extra:
            e.update(extra)
        return e

    def gemv_case(key, m, n, k, fmt, group, outliers):
        ws = weight_copies(fmt, n, k, group)
        x = acts(m, k, *(outliers or (0, 0)))
        y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
        fns = [lambda c=c: wq.wq_w4a16_gemv(x, n, fmt, group, *c, out=y) for c in ws]
        us, clk = _timed_launches(fns, sampler)
        nb = packed_bytes(fmt, n, k, group) + 2 * m * k + 2 * m * n
        out[key].append(entry("%s M=%d %dx%d" % ("nf4-b64" if fmt == NF else "int4-g%d" % group,
                                                 m, n, k), us, clk, nb, 2 * m * n * k,
                              extra={"weight_copies": len(ws)}))
        del ws, fns

    with ClockSampler(torch.cuda.current_device(), period=0.01) as sampler:
        # 1: the tiny GEMV
        gemv_case("config1_gemv_tiny", 1, 1024, 1024, F, 64, None)
        # 2: NF4 dequantization
        for n, k in [(28672, 8192), (8192, 8192), (5120, 25600)]:
            cw, am, _ = wq.wq_quantize_pack(NF, normal(n, k, std=0.02), 64)
            r = _copies_for(n * k // 2 + n * k // 16)
            sets = [(cw, am)] + [(cw.clone(), am.clone()) for _ in range(r - 1)]
            o = torch.empty(n * k, dtype=torch.bfloat16, device=device)
            fns = [lambda c=c: wq.wq_nf4_dequant(c[0], c[1], n * k, out=o) for c in sets]
            us, clk = _timed_launches(fns, sampler)
            out["config2_nf4_dequant"].append(entry("%dx%d" % (n, k), us, clk,
                                                    n * k * (0.5 + 4 / 64 + 2), 0))
            del sets, fns, o, cw, am
            torch.cuda.empty_cache()
        # 3: decode GEMV
        for n, k in [(4096, 4096), (11008, 4096), (4096, 11008)]:
            for fmt, group in ((F, 128), (NF, 64)):
                for m in (1, 4, 8, 16):
                    gemv_case("config3_gemv", m, n, k, fmt, group, (0.01, 20.0))
            torch.cuda.empty_cache()
        # 4: prefill GEMM beside dequantize-then-cuBLAS
        for n, k in [(4096, 4096), (14336, 4096), (4096, 14336)]:
            ws = weight_copies(F, n, k, 128)
            wd = torch.empty(n, k, dtype=torch.bfloat16, device=device)
            for m in (512, 2048, 8192):
                x = acts(m, k, 0, 0)
                y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
                wsp = wq.gemm_workspace(m, n, k, 128, device)
                fused = [lambda c=c: wq.wq_w4a16_gemm(x, n, F, 128, *c, workspace=wsp, out=y)
                         for c in ws]
                us, clk = _timed_launches(fused, sampler)

                def deq_mm(c):
                    wq.wq_int4_dequant(c[0], c[1], c[2], n, k, 128, out=wd)
                    torch.matmul(x, wd.t(), out=y)
                us_c, _ = _timed_launches([lambda c=c: deq_mm(c) for c in ws], sampler)
                nb = packed_bytes(F, n, k, 128) + 2 * m * k + 2 * m * n
                out["config4_gemm"].append(entry(
                    "int4-g128 M=%d %dx%d" % (m, n, k), us, clk, nb, 2 * m * n * k,
                    extra={"dequant_then_cublas_us": round(us_c, 2),
                           "fused_speedup": round(us_c / us, 3), "weight_copies": len(ws)}))
                del x, y, wsp, fused
            del ws, wd
            torch.cuda.empty_cache()
        # 5: MSD GEMM (and the fused GEMM on the same g128 layer at M >= 128)
        for n, k in [(5120, 5120), (25600, 5120), (5120, 25600)]:
            for group in (k, 128):
                ws = weight_copies(F, n, k, group)
                for m in (1, 16, 128, 1024):
                    x = acts(m, k, 0.005, 50.0)
                    y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
                    wsp = wq.msd_workspace(m, n, k, group, 2, device)
                    fns = [lambda c=c: wq.wq_msd_gemm(x, n, 2, group, *c, workspace=wsp, out=y)
                           for c in ws]
                    us, clk = _timed_launches(fns, sampler)
                    nb = packed_bytes(F, n, k, group) + 2 * m * k + 2 * m * n
                    tag = "per-channel" if group == k else "g128"
                    out["config5_msd"].append(entry("C=2 %s M=%d %dx%d" % (tag, m, n, k), us, clk,
                                                    nb, 2 * 2 * m * n * k, int8=True,
                                                    extra={"weight_copies": len(ws)}))
                    if group == 128 and m >= 128:
                        gws = wq.gemm_workspace(m, n, k, 128, device)
                        fused = [lambda c=c: wq.wq_w4a16_gemm(x, n, F, 128, *c, workspace=gws,
                                                              out=y) for c in ws]
                        us_f, _ = _timed_launches(fused, sampler)
                        out["msd_vs_fused_gemm"].append({
                            "case": "g128 M=%d %dx%d" % (m, n, k), "msd_us": round(us, 2),
                            "fused_gemm_us": round(us_f, 2), "msd_over_fused": round(us / us_f, 3)})
                        del gws, fused
                    if m == 128:
                        out["msd_accuracy"].append(dict(
                            case="%s M=128 %dx%d" % (tag, n, k),
                            **msd_accuracy(wq, x, n, k, group, ws[0], y, device)))
                    del x, y, wsp, fns
                del ws
                torch.cuda.empty_cache()
        # the MX path ("Multi-Scale Dequant...", Abstract): MXFP4 weights with
        # two MXFP4 activation passes, and one MXFP8 pass as the comparator,
        # decode sizes on the same Qwen3-32B shapes
        for n, k in [(5120, 5120), (25600, 5120), (5120, 25600)]:
            one = wq.wq_mx_quantize(normal(n, k, std=0.02))
            nb = n * k // 2 + n * k // 32
            ws = [one] + [tuple(t.clone() for t in one) for _ in range(_copies_for(nb) - 1)]
            for m in (1, 16):
                x = acts(m, k, 0.005, 50.0)
                y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
                for passes in (2, 1):
                    wsp = wq.mx_workspace(m, n, k, passes, device)
                    fns = [lambda c=c: wq.wq_mx_gemv(x, n, passes, *c, workspace=wsp, out=y)
                           for c in ws]
                    us, clk = _timed_launches(fns, sampler)
                    out["mx_msd_decode"].append(entry(
                        "%s M=%d %dx%d" % ("two MXFP4 passes" if passes == 2 else "one MXFP8 pass",
                                           m, n, k),
                        us, clk, nb + 2 * m * k + 2 * m * n, 2 * passes * m * n * k, fp8=True,
                        extra={"weight_copies": len(ws)}))
                del x, y
            del ws
            torch.cuda.empty_cache()
        # NF4 weights on the MSD path (integer codebook digits), decode sizes
        for n, k in [(5120, 5120), (25600, 5120), (5120, 25600)]:
            one = wq.wq_quantize_pack(NF, normal(n, k, std=0.02), 64)[:2]
            nb = n * k // 2 + n * k // 16
            ws = [one] + [tuple(t.clone() for t in one) for _ in range(_copies_for(nb) - 1)]
            for m in (1, 16):
                x = acts(m, k, 0.005, 50.0)
                y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
                wsp = wq.msd_workspace(m, n, k, 64, 2, device)
                fns = [lambda c=c: wq.wq_msd_gemm_nf4(x, n, 2, *c, workspace=wsp, out=y)
                       for c in ws]
                us, clk = _timed_launches(fns, sampler)
                out["nf4_msd_decode"].append(entry(
                    "C=2 M=%d %dx%d" % (m, n, k), us, clk, nb + 2 * m * k + 2 * m * n,
                    2 * 2 * 2 * m * n * k, int8=True,
                    extra={"weight_copies": len(ws), "ops": "int8 MMAs: 2 planes x 2 weight digits"}))
                del x, y, wsp
            del ws
            torch.cuda.empty_cache()
        # MSD decode attention over an INT4 KV cache ("Multi-Scale Dequant...",
        # Abstract: the cache is never dequantized), Qwen3-32B heads, beside
        # torch's scaled-dot-product attention on a bf16 cache of the same shape
        hq, hkv, d = 64, 8, 128
        for b, length in ((32, 8192), (8, 32768)):
            cache = [wq.kv_quantize_keys(normal(b, hkv, length, d, std=0.5)),
                     wq.kv_quantize_values(normal(b, hkv, length, d))]
            nb = 2 * b * hkv * length * (d // 2 + 4)          # codes + fp16 scale and zero
            copies = [cache] + [[tuple(t.clone() for t in kv) for kv in cache]
                                for _ in range(_copies_for(nb) - 1)]
            q = normal(b, hq, d).to(torch.bfloat16)
            o = torch.empty(b, hq, d, dtype=torch.bfloat16, device=device)
            wsp = wq.attention_workspace(b, hq, hkv, length, d, 2, device)
            fns = [lambda c=c: wq.wq_msd_decode_attention(q, c[0], c[1], 2, workspace=wsp, out=o)
                   for c in copies]
            us, clk = _timed_launches(fns, sampler)
            del copies, cache, fns
            torch.cuda.empty_cache()
            kb = normal(b, hkv, length, d).to(torch.bfloat16)
            vb = normal(b, hkv, length, d).to(torch.bfloat16)
            q4 = q.view(b, hq, 1, d)
            sdpa = [lambda: torch.nn.functional.scaled_dot_product_attention(
                q4, kb, vb, enable_gqa=True)]
            us_ref, _ = _timed_launches(sdpa, sampler)
            nb_ref = 2 * b * hkv * length * d * 2
            del kb, vb, sdpa
            torch.cuda.empty_cache()
            out["kv_msd_decode_attention"].append(entry(
                "C=2 B=%d L=%d Hq=%d Hkv=%d D=%d" % (b, length, hq, hkv, d), us, clk,
                nb + 2 * 2 * b * hq * d, 2 * 2 * 2 * 2 * b * hq * length * d, int8=True,
                extra={"sdpa_bf16_cache_us": round(us_ref, 2),
                       "sdpa_bf16_cache_gbs": round(nb_ref / (us_ref * 1e-6) / 1e9, 1),
                       "speedup_vs_sdpa_bf16": round(us_ref / us, 3),
                       "cache_bytes_int4": nb, "cache_bytes_bf16": nb_ref}))
            del q, o, wsp
            torch.cuda.empty_cache()
    return out


def msd_accuracy(wq, x, n, k, group, w, y, device, rows=64, cols=512):
    """Relative L2 errors, on sampled outputs, of the MSD product (C = 2) and
    of the bf16 dequantize-then-cuBLAS product against the exact product
    x . ((q - z) s)^T in fp64 (the codes from wq_unpack, the fp16 scales and
    zeros widened exactly; fp64 cuBLAS on the GPU). "Multi-Scale Dequant...",
    Abstract, reports lower L2 error than dequantization baselines in many
    settings but prints no numbers: this is a measurement, not a parity
    check."""
    qw, sc, zr = w
    m = x.shape[0]
    gen = torch.Generator(device="cpu").manual_seed(n + k + group)
    ri = torch.randperm(m, generator=gen)[:rows].to(device)
    ci = torch.randperm(n, generator=gen)[:cols].to(device)
    codes = wq.wq_unpack(wq.WQ_FMT_INT4_ASYM, qw, n, k).view(n, k)[ci].double()  # [cols, k]
    s64 = sc[ci].double().repeat_interleave(group, dim=1)
    z64 = zr[ci].double().repeat_interleave(group, dim=1)
    exact = x[ri].double() @ ((codes - z64) * s64).t()
    ws = wq.msd_workspace(m, n, k, group, 2, device)
    y_msd = wq.wq_msd_gemm(x, n, 2, group, qw, sc, zr, workspace=ws, out=y)[ri][:, ci].double()
    wd = wq.wq_int4_dequant(qw, sc, zr, n, k, group)
    y_deq = torch.matmul(x, wd.t())[ri][:, ci].double()
    nrm = exact.norm()
    return {"rel_l2_msd_c2": float((y_msd - exact).norm() / nrm),
            "rel_l2_bf16_dequant_cublas": float((y_deq - exact).norm() / nrm),
            "sample": "%d rows x %d cols" % (rows, cols)}


def run_gpu(args, rank, world, device):
    from bit_weight_quantized_weights_b200 import binding as wq
    peaks = load_peaks()
    step = Step(wq, device)
    ops = step.ops()

    for _ in range(args.warmup):
        for _, fn in ops:
            fn()
    st, detail = wq.wq_device_error()
    if st != wq.WQ_OK:
        raise RuntimeError("device error word set during warm-up: 0x%x" % detail)

    # per-op events inside the timed steps. By default the K timed steps
    # (with their per-op events, recorded as graph nodes) are captured once as
    # a CUDA graph and replayed as the timed region: the same launches in the
    # same order on fresh inputs, without the host's per-launch cost between
    # them. --eager launches them one by one instead.
    graph = None
    ev = {name: [(torch.cuda.Event(enable_timing=True, external=not args.eager),
                  torch.cuda.Event(enable_timing=True, external=not args.eager))
                 for _ in range(args.steps)] for name, _ in ops}

    def timed_steps():
        for i in range(args.steps):
            for name, fn in ops:
                a, b = ev[name][i]
                a.record()
                fn()
                b.record()

    if not args.eager:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            timed_steps()
        graph.replay()  # untimed: uploads the graph
        torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device(), period=0.005) as clocks:
        t0.record()
        if graph is not None:
            graph.replay()
        else:
            timed_steps()
        t1.record()
        torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = t0.elapsed_time(t1)
    elapsed_ms = max_over_ranks(elapsed_ms, world, device)
    per_op_ms = {name: sum(a.elapsed_time(b) for a, b in ev[name]) / args.steps for name, _ in ops}
    st, detail = wq.wq_device_error()
    if st != wq.WQ_OK:
        raise RuntimeError("device error word set during timing: 0x%x" % detail)

    # the tensor peak that matches this run's clocks (the same on every rank:
    # each rank's own record decides, and the value is summed over ranks)
    clk = clocks.summary()
    tf16, peak_kind = tensor_peak(peaks, clk)
    table = op_table(peaks, tf16)

    comparator = dequant_then_cublas(wq, step, per_op_ms["gemm"], args.warmup) if rank == 0 else None
    next_rows = None
    if rank == 0 and args.next_rows:
        next_rows = {"decdec": measure_decdec(
            wq, peaks, device, with_oracle=world == 1 and not args.no_cpu_baseline)}
    per_config = measure_per_config(wq, peaks, device) if rank == 0 and args.per_config else None

    ms_per_step = elapsed_ms / args.steps
    value = job_value(table, ms_per_step, world)

    # dominant kernel: the op with the largest share of the step
    dom = max(per_op_ms, key=per_op_ms.get)
    d = table[dom]
    dur_s = per_op_ms[dom] * 1e-3
    other = {}
    if d["bound"] == "tensor":
        achieved = d["flops"] / dur_s / 1e12
        peak = d["peak_flops"] / 1e12
        unit = "TFLOP/s" if dom == "gemm" else "TOP/s"
        mult = 1.0 if dom == "gemm" else 2.0
        other = {"frac_burst": round(achieved / (mult * peaks["bf16_tflops"]), 4),
                 "frac_sustained": round(achieved / (mult * peaks["bf16_tflops_sustained"]), 4)}
    else:
        achieved = d["bytes"] / dur_s / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    traffic = captured_traffic(dom)

    e2e = measure_e2e(args, step, ops, table, world, device) if args.e2e else None

    details = {name: dict(ms=per_op_ms[name], roof_ms=table[name]["t_roof"] * 1e3,
                          frac=table[name]["t_roof"] * 1e3 / per_op_ms[name],
                          gbs=table[name]["bytes"] / (per_op_ms[name] * 1e-3) / 1e9,
                          tflops=table[name]["flops"] / (per_op_ms[name] * 1e-3) / 1e12)
               for name in per_op_ms}
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4/nf4 weights, bf16 activations; fp16 and int8 tensor-core MMA, fp32 accumulate",
        "data": "synthetic (seeded; W ~ N(0,0.02) quantized on the GPU, x ~ N(0,1) with outlier channels)",
        "config": {"workload": "hot-path step, in this order: gemv int4-g128 and nf4-b64 M=16 "
                               "11008x4096; msd C=2 g128 M=16 25600x5120; nf4_dequant "
                               "28672x8192; gemm int4-g128 8192x14336x4096; msd C=2 g128 "
                               "M=1024 25600x5120",
                   "l2": "weights cold: each op has its own weights, last touched a step "
                         "earlier with the 600 MB NF4 stream (>4x L2) in between; activations "
                         "of the decode ops (<= 164 KB) may be L2-warm",
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "timing": ("eager launches" if args.eager else
                              "the K timed steps replayed as one captured CUDA graph") +
                             ", per-op CUDA events inside, device time"},
        "roofline": dict({"bound": d["bound"], "kernel": dom, "achieved": round(achieved, 2),
                          "peak": round(peak, 1), "unit": unit, "frac": round(achieved / peak, 4),
                          "traffic": traffic,
                          "peak_source": peaks["source"] + (
                              " (HBM copy)" if d["bound"] == "hbm" else
                              " (%s bf16, chosen by this run's clocks%s)"
                              % (peak_kind, "" if dom == "gemm" else "; x 2 for int8"))},
                         **other),
        "per_op": {k: {a: round(b, 4) for a, b in v.items()} for k, v in details.items()},
        "comparator": comparator,
        "next_rows": next_rows,
        "gpu_launches": Step.LAUNCHES_PER_STEP * args.steps,
        "clocks": clk,
        "tensor_peak": {"kind": peak_kind, "bf16_tflops": tf16,
                        "rule": "burst unless the timed region saw sw_power_cap or a median SM "
                                "clock below 0.9 x max"},
        "per_config": per_config,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(peaks, tf16=tf16)
    return line


def measure_e2e(args, step, ops, table, world, device):
    """The same step through the same C-ABI calls, but with every op's inputs
    in pinned host memory and its outputs read back to pinned host memory,
    all of the copies inside the timed region."""
    ins = {"nf4_dequant": [step.nf4_codes, step.nf4_absmax], "gemv_int4": [step.gx],
           "gemv_nf4": [], "gemm": [step.px], "msd_m16": [step.sx16], "msd_m1024": [step.sx1024]}
    outs = {"nf4_dequant": step.nf4_out, "gemv_int4": step.gy_i, "gemv_nf4": step.gy_n,
            "gemm": step.py, "msd_m16": step.sy16, "msd_m1024": step.sy1024}
    host_in = {n: [t.cpu().pin_memory() for t in ts] for n, ts in ins.items()}
    host_out = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in outs.items()}
    h2d = sum(t.numel() * t.element_size() for ts in host_in.values() for t in ts)
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    steps = max(1, min(args.steps, 5))

    # Uploads, compute and read-backs run on three streams so that the two
    # PCIe directions and the kernels overlap: an op waits for its own inputs
    # only; its read-back starts as soon as it finished; a step's upload into
    # an op's input buffer waits for the previous step's use of that buffer,
    # and an op's next write of its output waits for the previous read-back.
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    names = [name for name, _ in ops]
    used = {n: None for n in names}    # compute of the previous step finished
    read = {n: None for n in names}    # read-back of the previous step finished

    def one():
        for name, fn in ops:
            with torch.cuda.stream(up):
                if used[name] is not None:
                    up.wait_event(used[name])
                for dev_t, h in zip(ins[name], host_in[name]):
                    dev_t.copy_(h, non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(up)
            comp.wait_event(landed)
            if read[name] is not None:
                comp.wait_event(read[name])
            fn()
            done = torch.cuda.Event()
            done.record(comp)
            used[name] = done
            with torch.cuda.stream(down):
                down.wait_event(done)
                host_out[name].copy_(outs[name], non_blocking=True)
                back = torch.cuda.Event()
                back.record(down)
            read[name] = back

    one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a.record(comp)
    up.wait_event(a)
    down.wait_event(a)
    for _ in range(steps):
        one()
    for n in names:
        comp.wait_event(read[n])
    b.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), world, device) / steps
    return {"value": round(job_value(table, ms, world), 3), "unit": UNIT,
            "ms_per_step": round(ms, 3), "steps": steps,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample of the step
# ---------------------------------------------------------------------------

class OracleSample:
    """The CPU oracle on a row sample of every op of the step.

    prepare() draws and quantizes the sampled inputs (not timed); run() times
    only the oracle's arithmetic and returns (cpu seconds, roofline seconds of
    the sampled work). `scale` shrinks every sample proportionally."""

    def __init__(self, peaks, scale=1.0, tf16=None):
        self.table = op_table(peaks, tf16 if tf16 is not None else peaks["bf16_tflops"])
        self.scale = scale
        self.frac = {"nf4_dequant": scale / 256, "gemv_int4": scale / 16,
                     "gemv_nf4": scale / 16, "gemm": max(1, round(16 * scale)) / 8192,
                     "msd_m16": scale / 16, "msd_m1024": max(1, round(4 * scale)) / 1024}

    def prepare(self):
        from oracle import formats
        from bit_weight_quantized_weights_b200 import workloads
        f = self.frac
        n, k = NF4_SHAPE
        w = workloads.weights(max(1, int(n * f["nf4_dequant"])), k, seed=1).numpy()
        self.nf4 = formats.nf4_quantize(w)
        gn, gk = GEMV_SHAPE
        w, x = workloads.layer(16, max(16, int(gn * f["gemv_int4"])), gk, seed=2,
                               outliers=(0.01, 20.0))
        self.gx = x.float().numpy()
        self.gi = formats.int4_quantize(w.numpy(), 128)
        self.gn = formats.nf4_quantize(w.numpy())
        m, pn, pk = GEMM_SHAPE
        w, x = workloads.layer(round(m * f["gemm"]), pn, pk, seed=3)
        self.px = x.float().numpy()
        self.pw = formats.int4_quantize(w.numpy(), 128)
        sn, sk = MSD_SHAPE
        w, x = workloads.layer(16, max(16, int(sn * f["msd_m16"])), sk, seed=4,
                               outliers=(0.005, 50.0))
        self.s16 = (x.float().numpy(), formats.int4_quantize(w.numpy(), 128))
        w, x = workloads.layer(round(1024 * f["msd_m1024"]), sn, sk, seed=5,
                               outliers=(0.005, 50.0))
        self.s1024 = (x.float().numpy(), formats.int4_quantize(w.numpy(), 128))
        return self

    def run(self):
        from oracle import formats, msd, products
        t0 = time.perf_counter()
        formats.nf4_dequant_bf16(*self.nf4)
        products.w4a16_int4(self.gx, *self.gi, 128)
        products.w4a16_nf4(self.gx, *self.gn, GEMV_SHAPE[1])
        products.w4a16_int4(self.px, *self.pw, 128)
        for xf, (q, s, z) in (self.s16, self.s1024):
            a, sa = msd.decompose(xf, 2)
            msd.msd_product(a, sa, q, s, z, 128)
        t_cpu = time.perf_counter() - t0
        roof = sum(self.table[name]["t_roof"] * fr for name, fr in self.frac.items())
        return t_cpu, roof

    def describe(self):
        f = self.frac
        return ("oracle (NumPy, fp64) on a sample of the step: %.4g of the NF4 rows, %.4g of the "
                "GEMV rows, %d of 8192 GEMM tokens, %.4g of the MSD M=16 rows, %d of 1024 MSD "
                "tokens; value = roofline time of that work / CPU time"
                % (f["nf4_dequant"], f["gemv_int4"], round(f["gemm"] * 8192), f["msd_m16"],
                   round(f["msd_m1024"] * 1024)))


def decdec_cpu_baseline():
    """The oracle's salient-channel correction for one decode step on the host
    cores: channel selection plus the k-column correction over all 11008 rows
    (the residual matrix built once beforehand, untimed)."""
    import numpy as np
    from oracle import decdec
    n, k = DECDEC_SHAPE
    rng = np.random.default_rng(0)
    rt = (rng.standard_normal((k, n)) * 1e-3).astype(np.float16)
    x = rng.standard_normal((1, k)).astype(np.float32)
    x[:, ::64] *= 20.0
    t0 = time.perf_counter()
    reps = 20
    for _ in range(reps):
        idx = decdec.select_salient(x, DECDEC_K)
        decdec.correction(x, rt, idx)
    t = (time.perf_counter() - t0) / reps
    return {"kind": "oracle", "cores": oracle_cores(),
            "sample": "select + correction of one M=1 step (%d channels x %d rows)" % (DECDEC_K, n),
            "select_and_correction_us": round(t * 1e6, 1)}


def oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        return int(max([p.get("num_threads", 1) for p in threadpool_info()] + [1]))
    except Exception:
        return os.cpu_count()


def cpu_baseline(peaks, scale=1.0, tf16=None):
    """The oracle as it stands, timed once on a bounded sample of the step."""
    sample = OracleSample(peaks, scale, tf16).prepare()
    t_cpu, roof = sample.run()
    return {"value": round(100.0 * roof / t_cpu, 6), "unit": UNIT, "cores": oracle_cores(),
            "kind": "oracle", "sample": sample.describe(), "cpu_seconds": round(t_cpu, 2)}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas: barrier + max of the timing only)
# ---------------------------------------------------------------------------

def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v, world, device):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


PROFILE_CASES = ("nf4", "gemv_int4", "gemv_int4_m1", "gemv_nf4", "gemm", "msd", "msd_m16",
                 "decdec", "mx_m16", "nf4_msd_m16", "kv_attn")


def profile_case(case, device):
    """One small case of one kernel, run twice (warm-up + the launch an ncu
    capture selects with -s 1 -c 1). Inputs exceed L2 except the GEMV, whose
    DRAM figures rely on ncu's cache flush between passes."""
    from bit_weight_quantized_weights_b200 import binding as wq
    g = torch.Generator(device=device)
    g.manual_seed(0)

    def normal(*shape, std=1.0):
        return torch.randn(*shape, generator=g, device=device) * std

    if case == "nf4":
        n, k = 8192, 8192
        cw, am, _ = wq.wq_quantize_pack(wq.WQ_FMT_NF4, normal(n, k, std=0.02), 64)
        out = torch.empty(n * k, dtype=torch.bfloat16, device=device)
        fn = lambda: wq.wq_nf4_dequant(cw, am, n * k, out=out)  # noqa: E731
    elif case in ("gemv_int4", "gemv_int4_m1", "gemv_nf4"):
        (n, k), m = GEMV_SHAPE, (1 if case == "gemv_int4_m1" else 16)
        fmt = wq.WQ_FMT_NF4 if case == "gemv_nf4" else wq.WQ_FMT_INT4_ASYM
        grp = 128 if fmt == wq.WQ_FMT_INT4_ASYM else 64
        pw = wq.wq_quantize_pack(fmt, normal(n, k, std=0.02), grp)
        x = normal(m, k).to(torch.bfloat16)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
        fn = lambda: wq.wq_w4a16_gemv(x, n, fmt, grp, *pw, out=y)  # noqa: E731
    elif case == "gemm":
        m, n, k = 4096, GEMM_SHAPE[1], GEMM_SHAPE[2]
        pw = wq.wq_quantize_pack(wq.WQ_FMT_INT4_ASYM, normal(n, k, std=0.02), 128)
        x = normal(m, k).to(torch.bfloat16)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
        ws = wq.gemm_workspace(m, n, k, 128, device)
        fn = lambda: wq.wq_w4a16_gemm(x, n, wq.WQ_FMT_INT4_ASYM, 128, *pw, workspace=ws,  # noqa
                                      out=y)
    elif case in ("msd", "msd_m16"):
        m, (n, k) = (1024 if case == "msd" else 16), MSD_SHAPE
        pw = wq.wq_quantize_pack(wq.WQ_FMT_INT4_ASYM, normal(n, k, std=0.02), 128)
        x = normal(m, k).to(torch.bfloat16)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
        ws = wq.msd_workspace(m, n, k, 128, 2, device)
        fn = lambda: wq.wq_msd_gemm(x, n, 2, 128, *pw, workspace=ws, out=y)  # noqa: E731
    elif case == "mx_m16":
        m, (n, k) = 16, MSD_SHAPE
        codes, scales = wq.wq_mx_quantize(normal(n, k, std=0.02))
        x = normal(m, k).to(torch.bfloat16)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
        ws = wq.mx_workspace(m, n, k, 2, device)
        fn = lambda: wq.wq_mx_gemv(x, n, 2, codes, scales, workspace=ws, out=y)  # noqa: E731
    elif case == "nf4_msd_m16":
        m, (n, k) = 16, MSD_SHAPE
        codes, absmax, _ = wq.wq_quantize_pack(wq.WQ_FMT_NF4, normal(n, k, std=0.02), 64)
        x = normal(m, k).to(torch.bfloat16)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
        ws = wq.msd_workspace(m, n, k, 64, 2, device)
        fn = lambda: wq.wq_msd_gemm_nf4(x, n, 2, codes, absmax, workspace=ws, out=y)  # noqa
    elif case == "kv_attn":
        # decode attention over an INT4 KV cache, Qwen3-32B heads, B = 32 x 8192 tokens
        b, length, hq, hkv, d = 32, 8192, 64, 8, 128
        kc = wq.kv_quantize_keys(normal(b, hkv, length, d, std=0.5))
        vc = wq.kv_quantize_values(normal(b, hkv, length, d))
        q = normal(b, hq, d).to(torch.bfloat16)
        o = torch.empty(b, hq, d, dtype=torch.bfloat16, device=device)
        ws = wq.attention_workspace(b, hq, hkv, length, d, 2, device)
        fn = lambda: wq.wq_msd_decode_attention(q, kc, vc, 2, workspace=ws, out=o)  # noqa
    elif case == "decdec":
        # select, then the corrected GEMV (ncu -k regex:gemv_kernel captures it)
        (n, k), m = DECDEC_SHAPE, 1
        w = normal(n, k, std=0.02)
        pw = wq.wq_quantize_pack(wq.WQ_FMT_INT4_ASYM, w, 128)
        rt = wq.wq_residual(wq.WQ_FMT_INT4_ASYM, w, 128, *pw)
        x = normal(m, k).to(torch.bfloat16)
        idx = torch.empty(DECDEC_K, dtype=torch.int32, device=device)
        y = torch.empty(m, n, dtype=torch.bfloat16, device=device)

        def fn():
            wq.wq_select_salient(x, DECDEC_K, out=idx)
            wq.wq_w4a16_gemv_corrected(x, n, wq.WQ_FMT_INT4_ASYM, 128, *pw, rt, idx, out=y)
    else:
        raise SystemExit("unknown case %r (one of %s)" % (case, ", ".join(PROFILE_CASES)))
    for _ in range(2):
        fn()
        torch.cuda.synchronize()
    st, detail = wq.wq_device_error()
    if st != wq.WQ_OK:
        raise SystemExit("device error word 0x%x" % detail)
    print("case %s ok" % case)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="wq", choices=["wq", "reference"])
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", dest="next_rows", action="store_false",
                    help="skip the widening measurements timed after the step")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="skip the per-config throughput of every workload, timed after the step")
    ap.add_argument("--eager", action="store_true",
                    help="launch the timed steps one by one instead of replaying them as a "
                         "captured CUDA graph")
    ap.add_argument("--detail", default=None, help="also write the JSON line to this file")
    ap.add_argument("--case", default=None, choices=PROFILE_CASES,
                    help="run one small profiling case of one kernel and exit")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        peaks = load_peaks()
        steps = max(1, args.steps)
        sample = OracleSample(peaks, scale=0.25).prepare()
        for _ in range(args.warmup):
            sample.run()
        t_tot, roof_tot = 0.0, 0.0
        for _ in range(steps):
            t, r = sample.run()
            t_tot += t
            roof_tot += r
        value = round(100.0 * roof_tot / t_tot, 6)
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
                "steps": steps, "warmup": args.warmup, "ms_per_step": round(1e3 * t_tot / steps, 1),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic (seeded)",
                "config": {"workload": "same hot-path step as the GPU arm; each step is a bounded "
                                       "row sample run by the CPU oracle on the host cores"},
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_cores(),
                                 "kind": "oracle", "sample": sample.describe()},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if args.case:
        profile_case(args.case, device)
        return
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        line = run_gpu(args, rank, world, device)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if rank == 0:
        s = json.dumps(line)
        print(s)
        if args.detail:
            with open(args.detail, "w") as f:
                f.write(s + "\n")


if __name__ == "__main__":
    main()
