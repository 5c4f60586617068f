"""Benchmark of the NVFP4 W4A4 linear layer on B200.

One step = one pass of the hot path over one batch: dynamic activation
global scale (amax), activation quantisation, block-scaled FP4 GEMM with its
fused epilogue.  Weights are quantised once before timing (offline).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Prints one JSON line (rank 0).  The default workload is the largest
single-GPU configuration, the fused GDN input projection X[32768,5120] x
W[12352,5120] (six segments with their own global scales, gate epilogues);
the same line also carries the standalone quantiser on X[32768,17408]
(`kernels.quantize_32768x17408`, the metric's GB/s half).  `--impl reference`
times the CPU oracle on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4 GEMM TFLOPS & % dense-FP4 peak; quantize GB/s & % HBM peak (1 B200)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_PER_BF16 = 4.0  # nominal dense ratio: 9 PF FP4 / 2.25 PF BF16
NOMINAL_FP4_TFLOPS = 9000.0  # B200 datasheet dense FP4 (not measured here)
ROTATE = 4          # rotating input sets so consecutive steps miss in L2
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# dominant kernel, from one ncu capture of the kernel as it is now (the
# commands are in profiles/); an entry is removed when its kernel changes,
# until it is captured again.  "quant": both passes, captured on X[8192, 17408]
# and scaled by 4 rows-wise (the traffic grows with the rows).  "gdnrec": both
# recurrence launches, captured at full length (one pass each).
TRAFFIC_BYTES = {
    "actstats": 339345408,
    "gdnrec": 4052776533,
    "decode1": 50362112,
    "decode64": 50916352,
    "decode8": 50420224,
    "gdn": 1135872000,
    "kvfp8": 73506560,
    "mlp": 378899712,
    "oproj": 28804864,
    "quant": 2563600000,
    "requant": 36475136,
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        hi = max(sm) if sm else 0
        loaded = [s for s in sm if s >= 0.5 * hi] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------- distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world, backend=None):
    """Process group for N > 1 replicas: NCCL on GPUs (gloo for host-only runs
    of the timing plumbing).  Replicas exchange only the timing maximum and
    barriers; the path itself has no collective."""
    if world <= 1:
        return None
    import datetime
    import torch
    import torch.distributed as dist
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def tensor_peak(peaks: dict, chain_ms: float, clock_reasons) -> tuple:
    """The dense-FP4 roofline denominator (TFLOP/s) and its regime: a measured
    BF16 figure times the nominal FP4/BF16 ratio, the burst figure for a
    short chain of launches, the sustained one when the chain lasts a second
    or more or the sampled clocks show the power cap (a kernel timed inside a
    long run)."""
    sustained = chain_ms >= 1000.0 or "sw_power_cap" in (clock_reasons or [])
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    return float(peaks[key]) * FP4_PER_BF16, ("sustained" if sustained else "burst")


def e2e_choice(ms_pipelined: float, ms_serial: float) -> tuple:
    """The faster of the two end-to-end forms: (ms per step, mode)."""
    return (ms_pipelined, "pipelined") if ms_pipelined <= ms_serial else (ms_serial, "serial")


def dist_max(dist, value: float, device) -> float:
    """Max over ranks (device-timed milliseconds)."""
    if dist is None:
        return value
    import torch
    if dist.get_backend() == "gloo":
        device = "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(dist):
    if dist is not None:
        dist.barrier()


# ----------------------------------------------------------------- workloads

def workload_spec(name: str):
    from bit_quantized_linear_nvfp4_b200 import workloads as wl
    table = {"oproj": wl.OPROJ, "mlp": wl.MLP, "gdn": wl.GDN, "tiny": wl.TINY,
             "decode1": wl.DECODE[0], "decode8": wl.DECODE[1], "decode64": wl.DECODE[2]}
    if name == "quant":
        return None
    return table[name]


class ProductStep:
    """Device buffers for ROTATE input sets and CUDA graphs of the two stages."""

    def __init__(self, name: str, device, rows=None):
        import torch
        from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
        from bit_quantized_linear_nvfp4_b200 import workloads as wl
        self.nv, self.torch = nv, torch
        self.name = name
        self.device = device
        self.w = workload_spec(name)
        if self.w is None:
            M, K = wl.QUANT_SHAPE
            M = M if rows is None else rows  # a smaller case of the same kernels (profiling)
            x_np = wl.make_quant_input(rows=M)
            self.M, self.K, self.N = M, K, 0
            self.flops = 0.0
            self.sets = [self._act_set(x_np)]  # 1.14 GB input, larger than L2
            self.rotate = 1
            return
        w = self.w
        if rows is not None and not name.startswith("decode"):
            # the first `rows` rows of the same workload (a smaller case of the
            # same kernels, for profiler captures)
            import dataclasses
            w = self.w = dataclasses.replace(w, M=rows)
        self.M, self.K, self.N = w.M, w.K, w.N
        self.flops = w.flops()
        x_np = wl.make_x(w)
        segs = wl.make_w_segments(w)
        bounds = np.concatenate([[0], np.cumsum([s.width for s in w.segments])]).astype(np.int64)
        wdt = torch.float32 if w.dtype == "f32" else torch.bfloat16
        w_dev = torch.from_numpy(np.concatenate(segs)).to(device).to(wdt)
        self.W, self.gw = nv.nvfp4_quantize_segments(w_dev, bounds)
        del w_dev
        self.a_log = self.dt_bias = None
        if w.heads:
            a_log, dt_bias = wl.make_gate_params(w)
            self.a_log = torch.from_numpy(a_log).to(device)
            self.dt_bias = torch.from_numpy(dt_bias).to(device)
        self.bounds = bounds
        # rotate weights too for the weight-streaming (decode) shapes
        # decode shapes stream 50 MB weights: 8 copies (400 MB) keep back-to-back
        # launches from hitting the 126 MB L2
        self.rotate = 2 * ROTATE if name.startswith("decode") else ROTATE
        self.wsets = [(self.W, self.gw)]
        if name.startswith("decode"):
            for _ in range(self.rotate - 1):
                Wc = nv.Operand(self.W.codes.clone(), self.W.sf.clone(), self.W.rows, self.W.K)
                self.wsets.append((Wc, self.gw))
        self.sets = [self._act_set(x_np) for _ in range(self.rotate)]
        for i, s in enumerate(self.sets):
            s["W"], s["gw"] = self.wsets[i % len(self.wsets)]
            s["segs"] = self._segments(s)

    def _act_set(self, x_np):
        torch, nv = self.torch, self.nv
        dt = torch.float32 if (self.w is not None and self.w.dtype == "f32") else torch.bfloat16
        x = torch.from_numpy(x_np).to(self.device).to(dt)
        M, K = x.shape
        s = {
            "x": x,
            "codes": torch.empty((M, K // 2), dtype=torch.uint8, device=self.device),
            "sf": torch.empty(nv.nvfp4_sf_bytes(M, K), dtype=torch.uint8, device=self.device),
            "g": torch.empty(1, dtype=torch.float32, device=self.device),
            # calibrated static activation scale for the one-pass leg (set in capture())
            "gs": torch.empty(1, dtype=torch.float32, device=self.device),
            "ws": torch.empty(nv.nvfp4_quantize_workspace_bytes(1), dtype=torch.uint8, device=self.device),
        }
        s["A"] = nv.Operand(s["codes"], s["sf"], M, K)
        return s

    def _segments(self, s):
        torch, nv = self.torch, self.nv
        w = self.w
        outs, segs = [], []
        for i, seg in enumerate(w.segments):
            b0, b1 = int(self.bounds[i]), int(self.bounds[i + 1])
            if seg.epilogue == "swiglu_up":
                segs.append(nv.Segment(b0, b1, "swiglu_up"))
                continue
            kind = {"identity": "identity_f32" if w.out_dtype == "f32" else "identity_bf16",
                    "sigmoid": "sigmoid", "gdn_decay": "gdn_decay", "swiglu_gate": "swiglu_gate"}[seg.epilogue]
            dt = torch.bfloat16 if kind in ("identity_bf16", "swiglu_gate") else torch.float32
            out = torch.empty((self.M, b1 - b0), dtype=dt, device=self.device)
            outs.append(out)
            extra = {}
            if kind == "gdn_decay":
                extra = dict(A_log=self.a_log, dt_bias=self.dt_bias)
            segs.append(nv.Segment(b0, b1, kind, out, **extra))
        s["outs"] = outs
        return segs

    # stage launches (all work in libnvfp4)
    def quantize(self, s):
        self.nv.nvfp4_quantize(s["x"], codes=s["codes"], sf=s["sf"], g_out=s["g"], workspace=s["ws"])

    def gemm(self, s):
        self.nv.nvfp4_fused_proj(s["A"], s["g"], s["W"], s["gw"], s["segs"])

    def linear(self, s):
        # the whole layer in one call: quantise x, then the fused projection
        self.nv.nvfp4_linear(s["x"], s["W"], s["gw"], s["segs"], a_codes=s["codes"], a_sf=s["sf"],
                             g_a=s["g"], workspace=s["ws"])

    # one-pass forms: a calibrated static activation scale is given, so the
    # amax pass is skipped (quantiser alone, and the whole layer call)
    def quantize_static(self, s):
        self.nv.nvfp4_quantize(s["x"], s["gs"], codes=s["codes"], sf=s["sf"], g_out=s["g"])

    def linear_static(self, s):
        self.nv.nvfp4_linear(s["x"], s["W"], s["gw"], s["segs"], s["gs"], a_codes=s["codes"], a_sf=s["sf"],
                             g_a=s["g"])

    def launches_per_step(self):
        return 2 if self.w is None else 3  # amax, quantize (+ GEMM)

    def capture(self):
        torch = self.torch
        self.gq, self.gg, self.gl, self.gqs, self.gls = [], [], [], [], []
        for s in self.sets:  # warm the launch path once outside capture
            self.quantize(s)
            s["gs"].copy_(s["g"])  # "calibration": this input's own amax scale, fixed from here on
            self.quantize_static(s)
            if self.w is not None:
                self.gemm(s)
                self.linear(s)
                self.linear_static(s)
        torch.cuda.synchronize()

        def graph(fn, s):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn(s)
            return g

        for s in self.sets:
            self.gq.append(graph(self.quantize, s))
            self.gqs.append(graph(self.quantize_static, s))
            if self.w is not None:
                self.gg.append(graph(self.gemm, s))
                self.gl.append(graph(self.linear, s))
                self.gls.append(graph(self.linear_static, s))
        torch.cuda.synchronize()

    def step_graph(self, r):
        """One pass of the whole path: the layer call (or the quantiser alone)."""
        return self.gl[r] if self.w is not None else self.gq[r]

    def alg_bytes_quant(self):
        # amax pass reads X; the quantiser reads X and writes codes + scales
        esz = 4 if (self.w is not None and self.w.dtype == "f32") else 2
        e = self.M * self.K
        return {"amax": e * esz, "quantize": e * esz + e // 2 + e // 16}

    def alg_bytes_gemm(self):
        M, N, K = self.M, self.N, self.K
        out_bytes = 0
        for seg in self.w.segments:
            if seg.epilogue in ("identity",):
                out_bytes += M * seg.width * (4 if self.w.out_dtype == "f32" else 2)
            elif seg.epilogue in ("sigmoid", "gdn_decay"):
                out_bytes += M * seg.width * 4
            elif seg.epilogue == "swiglu_gate":
                out_bytes += M * seg.width * 2
        return M * K // 2 + M * K // 16 + N * K // 2 + N * K // 16 + out_bytes


def run_product(args):
    import torch
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = dist_init(world)
    peaks, peak_src = load_peaks()

    step = ProductStep(args.workload, device, rows=args.rows)
    step.capture()
    stream = torch.cuda.current_stream()
    K, Wm = args.steps, args.warmup
    R = len(step.sets)

    def staged(i, evs):
        # the two stages as separate calls, an event on each side of each
        r = i % R
        evs[0].record(stream)
        step.gq[r].replay()
        evs[1].record(stream)
        if step.w is not None:
            step.gg[r].replay()
        evs[2].record(stream)

    def chain(fn):
        # K calls of one stage over the rotating input sets, captured in one
        # CUDA graph: consecutive launches overlap prologue and tail through
        # programmatic dependent launch, as a model's layer sequence does
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(K):
                fn(step.sets[i % R])
        return g

    main = chain(step.linear if step.w is not None else step.quantize)
    for i in range(Wm):
        step.step_graph(i % R).replay()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    # timed region: K steps, each one pass of the path (the layer call), as
    # one graph replay
    dist_barrier(dist)
    torch.cuda.synchronize()
    t0.record(stream)
    main.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    dist_barrier(dist)
    # per-stage device times (dominant-kernel roofline), same inputs
    for i in range(min(Wm, 3)):
        staged(i, evs[i])
    torch.cuda.synchronize()
    for i in range(K):
        staged(i, evs[i])
    torch.cuda.synchronize()

    def chain_ms(fn):
        # K chained launches of one stage in one graph, after one warm-up replay
        g = chain(fn)
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / K

    # one-pass (calibrated static scale) forms beside the two-pass ones
    q1_ms = chain_ms(step.quantize_static)
    l1_ms = chain_ms(step.linear_static) if step.w is not None else None
    # each stage launched back to back K times (rotating inputs): the average
    # launch duration the roofline divides by; the isolated, event-bracketed
    # stage times are reported beside it
    qb2b_ms = chain_ms(step.quantize)
    gb2b_ms = chain_ms(step.gemm) if step.w is not None else None
    clk = clocks.stop()
    total_ms = t0.elapsed_time(t1)
    total_ms = dist_max(dist, total_ms, device)
    ms_step = total_ms / K
    q_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    g_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / K if step.w is not None else 0.0
    nv = step.nv
    nv.nvfp4_check()

    # end to end through host buffers: pinned X in, result out, every step
    # (at most 100 steps: each moves up to a GB over PCIe)
    e2e = measure_e2e(step, min(K, 100), min(Wm, 5), stream)
    # whole job: the slowest rank's time, every rank's work
    e2e_ms = dist_max(dist, e2e["ms_per_step"], device)
    e2e["value"] = e2e["value"] * e2e["ms_per_step"] / e2e_ms * world
    e2e["ms_per_step"] = e2e_ms
    for form in ("serial", "pipelined"):
        f_ms = dist_max(dist, e2e[form + "_ms_per_step"], device)
        e2e[form + "_value"] = e2e[form + "_value"] * e2e[form + "_ms_per_step"] / f_ms * world
        e2e[form + "_ms_per_step"] = f_ms

    qb = step.alg_bytes_quant()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    kernels = {"quantize_stage_ms": q_ms, "quantize_back_to_back_ms": qb2b_ms,
               "quantize_stage_gbs": (qb["amax"] + qb["quantize"]) / (q_ms * 1e-3) / 1e9,
               "quantize_stage_frac_hbm": (qb["amax"] + qb["quantize"]) / (q_ms * 1e-3) / 1e9 / hbm,
               "quantize_one_pass_ms": q1_ms,
               "quantize_one_pass_gbs": qb["quantize"] / (q1_ms * 1e-3) / 1e9,
               "quantize_one_pass_frac_hbm": qb["quantize"] / (q1_ms * 1e-3) / 1e9 / hbm}
    if l1_ms is not None:
        kernels["layer_one_pass_ms"] = l1_ms
        kernels["layer_two_pass_ms"] = ms_step
        kernels["layer_one_pass_tflops"] = step.flops / (l1_ms * 1e-3) / 1e12
    if step.w is not None and args.workload.startswith("decode"):
        # few tokens: the GEMM streams W from HBM, so its roofline is bandwidth
        gbs = step.alg_bytes_gemm() / (gb2b_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                "traffic": TRAFFIC_BYTES.get(args.workload), "peak_source": f"{peak_src} copy bandwidth",
                "kernel": "nvfp4 decode gemm (tcgen05 mxf4nvf4, split-K cluster)", "ms_per_launch": gb2b_ms,
                "ms_per_isolated_launch": g_ms}
    elif step.w is not None:
        # The denominator is a measured BF16 figure times the nominal dense
        # FP4/BF16 ratio: the burst figure when the GEMM's back-to-back chain
        # is short (tens of ms), the sustained one when the chain runs a
        # second or more or the clocks show the power cap (a kernel timed
        # inside a long run).  The nominal 9 PF and the other figure are
        # reported beside it.
        fp4_burst = float(peaks["bf16_tflops"]) * FP4_PER_BF16
        fp4_sustained = float(peaks["bf16_tflops_sustained"]) * FP4_PER_BF16
        fp4_peak, regime = tensor_peak(peaks, gb2b_ms * K, clk.get("reasons"))
        ach = step.flops / (gb2b_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": fp4_peak, "unit": "TFLOP/s",
                "frac": ach / fp4_peak, "traffic": TRAFFIC_BYTES.get(args.workload),
                "peak_source": f"{peak_src} {regime} bf16 x {FP4_PER_BF16:g} (nominal dense FP4/BF16)",
                "kernel": "nvfp4 gemm (tcgen05 mxf4nvf4)", "ms_per_launch": gb2b_ms,
                "ms_per_isolated_launch": g_ms, "frac_of_nominal_9pf": ach / NOMINAL_FP4_TFLOPS,
                "frac_of_burst_bf16_x4": ach / fp4_burst, "frac_of_sustained_bf16_x4": ach / fp4_sustained,
                "gemm_chain_ms": gb2b_ms * K}
    else:
        bytes_step = qb["amax"] + qb["quantize"]
        ach = bytes_step / (qb2b_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "traffic": TRAFFIC_BYTES.get(args.workload), "peak_source": f"{peak_src} copy bandwidth",
                "kernel": "nvfp4 amax + quantize", "ms_per_launch": qb2b_ms, "ms_per_isolated_launch": q_ms}
        value = bytes_step * world / (ms_step * 1e-3) / 1e9
        unit = "GB/s"
    if step.w is not None:  # prefill and decode: the metric is the layer's TFLOP/s
        kernels["gemm_ms"] = g_ms
        kernels["gemm_back_to_back_ms"] = gb2b_ms
        kernels["gemm_alg_bytes"] = step.alg_bytes_gemm()
        kernels["gemm_gbs"] = step.alg_bytes_gemm() / (gb2b_ms * 1e-3) / 1e9
        value = step.flops * world / (ms_step * 1e-3) / 1e12
        unit = "TFLOP/s"

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": K, "warmup": Wm,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "nvfp4", "data": "synthetic (seeded N(0,1) activations with outlier channels, N(0,0.02) weights)",
        "config": {"workload": step.name if step.w is None else step.w.name, "M": step.M, "N": step.N, "K": step.K,
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": f"{R} rotating input sets, {'weights rotated too, ' if args.workload.startswith('decode') else ''}"
                         "working set above the 126 MB L2" if R > 1 else "input larger than L2",
                   "launch": "the K timed steps are one CUDA graph of K chained layer calls (programmatic dependent "
                             "launch between kernels); dominant-kernel back-to-back times likewise"},
        "roofline": roof, "kernels": kernels, "clocks": clk, "e2e": e2e,
        "gpu_launches": step.launches_per_step() * K,
    }
    for g in step.gq + step.gg + step.gl + step.gqs + step.gls:
        del g
    if step.w is not None and not args.no_quant_line:
        # the metric's second half (quantiser GB/s) on its own workload, in
        # the same run; outside the timed region of the projection
        del step
        torch.cuda.empty_cache()
        kernels["quantize_32768x17408"] = measure_quantizer(device, K, Wm, hbm)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, target_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def measure_e2e(step, K, Wm, stream):
    """The layer end to end through the library's public call: every step
    copies the step's input from pinned host memory to the device, calls the
    C ABI (nvfp4_linear through the binding, or nvfp4_quantize for the
    quantiser workload; host validation, tensor-map encoding and launches
    included) and copies the results back to pinned host memory.

    The value is the pipelined form a serving loop runs: uploads on one
    stream, the library call on the launching stream, read-backs on a third,
    over two device buffer sets, so that step i+1's upload and step i-1's
    read-back overlap step i's call (events order every reuse of a buffer).
    The one-stream form, where each step's copies and call run in turn, is
    reported beside it."""
    import torch
    nb = min(2, len(step.sets))
    sets = step.sets[:nb]

    def outs_of(s):
        return s.get("outs") or [s["codes"]]

    x_host = sets[0]["x"].cpu().pin_memory()
    out_host = [o.cpu().pin_memory() for o in outs_of(sets[0])]
    h2d = x_host.numel() * x_host.element_size()
    d2h = sum(o.numel() * o.element_size() for o in out_host)
    call = step.linear if step.w is not None else step.quantize

    def one(replay=False):
        s = sets[0]
        s["x"].copy_(x_host, non_blocking=True)
        if replay:
            step.step_graph(0).replay()
        else:
            call(s)
        for dst, src in zip(out_host, outs_of(s)):
            dst.copy_(src, non_blocking=True)

    def timed(replay):
        for _ in range(Wm):
            one(replay)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K):
            one(replay)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / K

    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event() for _ in range(nb)] for k in ("h2d", "call", "d2h")}

    def pipe_step(i):
        bi = i % nb
        s = sets[bi]
        if i >= nb:
            s_in.wait_event(ev["call"][bi])  # the call of step i - nb has read x
        with torch.cuda.stream(s_in):
            s["x"].copy_(x_host, non_blocking=True)
            ev["h2d"][bi].record(s_in)
        stream.wait_event(ev["h2d"][bi])
        if i >= nb:
            stream.wait_event(ev["d2h"][bi])  # the results of step i - nb are read back
        with torch.cuda.stream(stream):
            call(s)
            ev["call"][bi].record(stream)
        s_out.wait_event(ev["call"][bi])
        with torch.cuda.stream(s_out):
            for dst, src in zip(out_host, outs_of(s)):
                dst.copy_(src, non_blocking=True)
            ev["d2h"][bi].record(s_out)

    def pipelined():
        for i in range(Wm):
            pipe_step(i)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_in.wait_event(a)
        s_out.wait_event(a)
        for i in range(K):
            pipe_step(i)
        stream.wait_event(ev["d2h"][(K - 1) % nb])  # the last read-back ends the step sequence
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / K

    ms_serial = timed(False)
    ms_graph = timed(True)
    ms = pipelined()
    # every set gets the same input, so the last read-back must equal the
    # device result it was copied from (a race would show here)
    last = outs_of(sets[(K - 1) % nb])
    if not all(torch.equal(h, d.cpu()) for h, d in zip(out_host, last)):
        raise RuntimeError("pipelined end-to-end read-back differs from the device result")

    def rate(t):
        if step.w is not None:
            return step.flops / (t * 1e-3) / 1e12
        qb = step.alg_bytes_quant()
        return (qb["amax"] + qb["quantize"]) / (t * 1e-3) / 1e9

    unit = "TFLOP/s" if step.w is not None else "GB/s"
    # the faster of the two forms is the value (for a few tokens the three
    # streams' host-side bookkeeping costs more than the overlap saves)
    best, mode = e2e_choice(ms, ms_serial)
    return {"value": rate(best), "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": best, "call": "nvfp4_linear" if step.w is not None else "nvfp4_quantize",
            "mode": mode,
            "pipeline": f"uploads, calls and read-backs on three streams over {nb} device buffer set(s)",
            "pipelined_value": rate(ms), "pipelined_ms_per_step": ms,
            "serial_value": rate(ms_serial), "serial_ms_per_step": ms_serial,
            "graph_replay_ms_per_step": ms_graph, "steps": K, "warmup": Wm}


def measure_quantizer(device, K, Wm, hbm):
    """The standalone quantiser on X[32768, 17408] BF16 (1.14 GB, larger than
    L2): amax + quantise (device-computed scale) and the one-pass form with a
    calibrated static scale, each launched back to back K times; GB/s of
    algorithmic bytes (2 B read per element per pass, 0.5 B codes and
    0.0625 B scales written) and the fraction of the measured HBM copy
    bandwidth."""
    import torch
    step = ProductStep("quant", device)
    step.capture()
    stream = torch.cuda.current_stream()

    def b2b(fn):
        # K chained launches in one CUDA graph, after one warm-up replay
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(K):
                fn(step.sets[0])
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / K

    dyn_ms = b2b(step.quantize)
    cal_ms = b2b(step.quantize_static)
    qb = step.alg_bytes_quant()
    dyn_gbs = (qb["amax"] + qb["quantize"]) / (dyn_ms * 1e-3) / 1e9
    cal_gbs = qb["quantize"] / (cal_ms * 1e-3) / 1e9
    out = {"shape": [step.M, step.K], "dynamic_ms": dyn_ms, "dynamic_gbs": dyn_gbs,
           "dynamic_frac_hbm": dyn_gbs / hbm, "calibrated_ms": cal_ms, "calibrated_gbs": cal_gbs,
           "calibrated_frac_hbm": cal_gbs / hbm, "alg_bytes_dynamic": qb["amax"] + qb["quantize"],
           "alg_bytes_calibrated": qb["quantize"], "launches_back_to_back": K,
           "kernels": "amax_kernel + quant_kernel (dynamic); quant_kernel (calibrated)"}
    for g in step.gq + step.gqs:
        del g
    del step
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------- CPU oracle

def _oracle_sample_step(name, rows, x_np, wq, g_a, extra):
    """One oracle pass over `rows` rows of the workload: quantise the rows,
    FP64 GEMM against the pre-quantised weights, epilogues."""
    from oracle import nvfp4_oracle as o
    aq = o.quantize(x_np[:rows], g_a)
    if wq is None:
        return
    w, segs_q, scales, epis, gate = extra
    o.fused_projection(aq, segs_q, scales, epis, gate)


def _prepare_oracle(name):
    from bit_quantized_linear_nvfp4_b200 import workloads as wl
    from oracle import nvfp4_oracle as o
    w = workload_spec(name)
    if w is None:
        x = wl.make_quant_input(rows=2048)
        return None, x, None, o.global_scale(x), None
    x = wl.make_x(w, rows=min(w.M, 4096))
    g_a = o.global_scale(x)
    segs = wl.make_w_segments(w)
    wq = [o.quantize(s) for s in segs]
    gate = wl.make_gate_params(w) if w.heads else None
    extra = (w, [(c, s) for c, s, _ in wq], [g for _, _, g in wq], [s.epilogue for s in w.segments], gate)
    return w, x, wq, g_a, extra


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(name, target_s=12.0, steps=None):
    """Time the oracle as it stands on a bounded row sample; throughput in the
    bench's unit scaled by the rows processed."""
    w, x, wq, g_a, extra = _prepare_oracle(name)
    K = x.shape[1]
    rows = 8
    t = time.perf_counter()
    _oracle_sample_step(name, rows, x, wq, g_a, extra)
    dt = max(time.perf_counter() - t, 1e-3)
    rows = int(min(x.shape[0], max(8, rows * (target_s / 2) / dt)))
    t = time.perf_counter()
    n = 0
    while True:
        _oracle_sample_step(name, rows, x, wq, g_a, extra)
        n += 1
        el = time.perf_counter() - t
        if el >= target_s * 0.5 or n >= 4:
            break
    per = el / n
    if w is not None:
        val = 2.0 * rows * w.N * K / per / 1e12
        unit = "TFLOP/s"
    else:
        val = rows * K * (2 + 2 + 0.5 + 0.0625) / per / 1e9
        unit = "GB/s"
    return {"value": val, "unit": unit, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{rows} rows of the workload per pass ({n} passes, {el:.1f} s): quantise rows + FP64 GEMM + epilogue"
                      if w is not None else f"{rows} rows x {K} per pass ({n} passes): amax + quantise",
            "host_cpus": os.cpu_count()}


def run_requant(args):
    """Checkpoint-side harmonisation of the GDN in-projection weight
    [12352, 5120] (six modules): nvfp4_requantize_segments under the fused
    tensor's scale, one call per step; HBM-bound (reads and writes codes and
    scale bytes)."""
    import torch
    from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
    from bit_quantized_linear_nvfp4_b200 import workloads as wl
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = dist_init(world)
    peaks, peak_src = load_peaks()
    w = wl.GDN
    segs = wl.make_w_segments(w)
    bounds = np.concatenate([[0], np.cumsum([sg.width for sg in w.segments])]).astype(np.int64)
    N, K = int(bounds[-1]), w.K
    wdev = torch.from_numpy(np.concatenate(segs)).to(device).to(torch.bfloat16)
    sets = []
    for _ in range(ROTATE):
        W, gw = nv.nvfp4_quantize_segments(wdev, bounds)
        out = (torch.empty_like(W.codes), torch.empty_like(W.sf), torch.empty_like(gw))
        sets.append((W, gw, out))
    del wdev
    stream = torch.cuda.current_stream()

    def call(i):
        W, gw, (c, sf, g) = sets[i % ROTATE]
        nv.nvfp4_requantize_segments(W, bounds, gw, codes=c, sf=sf, g_out=g)

    for i in range(ROTATE):
        call(i)
    torch.cuda.synchronize()
    graphs = []
    for i in range(ROTATE):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call(i)
        graphs.append(g)
    Kst, Wm = args.steps, args.warmup
    for i in range(Wm):
        graphs[i % ROTATE].replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(dist)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(Kst):
        graphs[i % ROTATE].replay()
    t1.record(stream)
    torch.cuda.synchronize()
    dist_barrier(dist)
    clk = clocks.stop()
    ms = dist_max(dist, t0.elapsed_time(t1), device) / Kst
    nv.nvfp4_check()
    per_set = N * K // 2 + nv.nvfp4_sf_bytes(N, K)
    bytes_step = 2 * per_set
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    ach = bytes_step / (ms * 1e-3) / 1e9
    # end to end: the checkpoint's codes and scales in from pinned host memory, the result out
    W0, gw0, (c0, sf0, g0) = sets[0]
    h_codes, h_sf = W0.codes.cpu().pin_memory(), W0.sf.cpu().pin_memory()
    o_codes, o_sf = torch.empty_like(h_codes).pin_memory(), torch.empty_like(h_sf).pin_memory()

    def e2e_one():
        W0.codes.copy_(h_codes, non_blocking=True)
        W0.sf.copy_(h_sf, non_blocking=True)
        graphs[0].replay()
        o_codes.copy_(c0, non_blocking=True)
        o_sf.copy_(sf0, non_blocking=True)

    for _ in range(Wm):
        e2e_one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(Kst):
        e2e_one()
    b.record(stream)
    torch.cuda.synchronize()
    ms_e2e = dist_max(dist, a.elapsed_time(b) / Kst, device)  # max over ranks
    line = {
        "metric": METRIC, "value": bytes_step * world / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": world,
        "steps": Kst, "warmup": Wm, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4 (FP32 arithmetic)", "data": "synthetic (N(0,0.02) weights, six modules)",
        "config": {"workload": "requant_gdn_weight_12352x5120", "N": N, "K": K, "segments": len(w.segments),
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": f"{ROTATE} rotating weight copies, working set above the 126 MB L2"},
        "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                     "traffic": TRAFFIC_BYTES.get("requant"), "peak_source": f"{peak_src} copy bandwidth",
                     "kernel": "nvfp4 requantize", "ms_per_launch": ms},
        "clocks": clk,
        "e2e": {"value": bytes_step * world / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": per_set,
                "d2h_bytes_per_step": per_set, "ms_per_step": ms_e2e},
        "gpu_launches": Kst,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import nvfp4_oracle as o
        rows = 512
        wq = [o.quantize(sg_w) for sg_w in segs]
        c_all = np.concatenate([c for c, _, _ in wq])[:rows]
        s_all = np.concatenate([sf for _, sf, _ in wq])[:rows]
        g_rows = np.repeat(np.array([g for _, _, g in wq], np.float32), [sg.width for sg in w.segments])[:rows]
        g_c = max(g for _, _, g in wq)
        t = time.perf_counter()
        n = 0
        while time.perf_counter() - t < args.cpu_seconds / 2 or n == 0:
            o.requantize(c_all, s_all, g_rows, g_c)
            n += 1
        per = (time.perf_counter() - t) / n
        line["cpu_baseline"] = {"value": 2 * rows * K * 0.5625 / per / 1e9, "unit": "GB/s", "cores": _blas_threads(),
                                "kind": "oracle", "sample": f"{rows} rows x {K} per pass ({n} passes)",
                                "host_cpus": os.cpu_count()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    for g in graphs:
        del g
    if dist is not None:
        dist.destroy_process_group()


def run_kvfp8(args):
    """FP8 (E4M3) KV-cache codec: quantise the K and V of a 32768-token prefill
    chunk (8 KV heads x 128, BF16) under calibrated static scales, two calls
    per step; HBM-bound (2 B read + 1 B written per element)."""
    import torch
    from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
    from bit_quantized_linear_nvfp4_b200 import workloads as wl
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = dist_init(world)
    peaks, peak_src = load_peaks()
    T, C = 32768, 1024
    rng = np.random.default_rng(6)
    kv_np = [wl.round_to_bf16(rng.standard_normal((T, C)).astype(np.float32)) for _ in range(2)]
    scales = [np.float32(np.abs(a).max() / 448) for a in kv_np]
    sets = []
    for r in range(ROTATE):
        srcs = [torch.from_numpy(a).to(device).to(torch.bfloat16) for a in kv_np]
        outs = [torch.empty((T, C), dtype=torch.uint8, device=device) for _ in range(2)]
        sc = [torch.tensor([v], dtype=torch.float32, device=device) for v in scales]
        sets.append((srcs, outs, sc))
    stream = torch.cuda.current_stream()

    def call(i):
        srcs, outs, sc = sets[i % ROTATE]
        for x, o_, s_ in zip(srcs, outs, sc):
            nv.nvfp4_kv_fp8_quantize(x, s_, out=o_)

    for i in range(ROTATE):
        call(i)
    torch.cuda.synchronize()
    graphs = []
    for i in range(ROTATE):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call(i)
        graphs.append(g)
    Kst, Wm = args.steps, args.warmup
    for i in range(Wm):
        graphs[i % ROTATE].replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(dist)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(Kst):
        graphs[i % ROTATE].replay()
    t1.record(stream)
    torch.cuda.synchronize()
    dist_barrier(dist)
    clk = clocks.stop()
    ms = dist_max(dist, t0.elapsed_time(t1), device) / Kst
    nv.nvfp4_check()
    bytes_step = 2 * T * C * 3
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    ach = bytes_step / (ms * 1e-3) / 1e9
    srcs0, outs0, _ = sets[0]
    h_in = [x.cpu().pin_memory() for x in srcs0]
    h_out = [torch.empty((T, C), dtype=torch.uint8).pin_memory() for _ in range(2)]

    def e2e_one():
        for d, h in zip(srcs0, h_in):
            d.copy_(h, non_blocking=True)
        graphs[0].replay()
        for h, d in zip(h_out, outs0):
            h.copy_(d, non_blocking=True)

    for _ in range(Wm):
        e2e_one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(Kst):
        e2e_one()
    b.record(stream)
    torch.cuda.synchronize()
    ms_e2e = dist_max(dist, a.elapsed_time(b) / Kst, device)  # max over ranks
    line = {
        "metric": METRIC, "value": bytes_step * world / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": world,
        "steps": Kst, "warmup": Wm, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8 e4m3 (FP32 arithmetic)", "data": "synthetic (N(0,1) BF16 K and V)",
        "config": {"workload": "kv_fp8_encode_2x32768x1024", "tokens": T, "cols": C, "tensors": 2,
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": f"{ROTATE} rotating K/V sets, working set above the 126 MB L2"},
        "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                     "traffic": TRAFFIC_BYTES.get("kvfp8"), "peak_source": f"{peak_src} copy bandwidth",
                     "kernel": "nvfp4 kv fp8 encode", "ms_per_launch": ms / 2},
        "clocks": clk,
        "e2e": {"value": bytes_step * world / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": 2 * T * C * 2,
                "d2h_bytes_per_step": 2 * T * C, "ms_per_step": ms_e2e},
        "gpu_launches": 2 * Kst,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import nvfp4_oracle as o
        rows = 2048
        t = time.perf_counter()
        n = 0
        while time.perf_counter() - t < args.cpu_seconds / 2 or n == 0:
            o.kv_fp8_quantize(kv_np[0][:rows], scales[0])
            n += 1
        per = (time.perf_counter() - t) / n
        line["cpu_baseline"] = {"value": rows * C * 3 / per / 1e9, "unit": "GB/s", "cores": _blas_threads(),
                                "kind": "oracle", "sample": f"{rows} rows x {C} per pass ({n} passes)",
                                "host_cpus": os.cpu_count()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    for g in graphs:
        del g
    if dist is not None:
        dist.destroy_process_group()


def run_actstats(args):
    """Activation statistics of the GDN prefill activation X[32768, 5120] (BF16,
    0.5% outlier channels x100): one nvfp4_activation_stats call per step, with
    the global scale for the A4 error; HBM-bound (2 B read per element)."""
    import torch
    from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
    from bit_quantized_linear_nvfp4_b200 import workloads as wl
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = dist_init(world)
    peaks, peak_src = load_peaks()
    w = wl.GDN
    x_np = wl.make_x(w)
    M, K = x_np.shape
    sets = []
    for _ in range(ROTATE):
        x = torch.from_numpy(x_np).to(device).to(torch.bfloat16)
        _, g = nv.nvfp4_quantize(x)
        acc = nv.nvfp4_activation_stats(x, g)
        sets.append((x, g, acc))
    stream = torch.cuda.current_stream()
    graphs = []
    torch.cuda.synchronize()
    for x, g, acc in sets:
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            nv.nvfp4_activation_stats(x, g, into=acc)
        graphs.append(gr)
    Kst, Wm = args.steps, args.warmup
    for i in range(Wm):
        graphs[i % ROTATE].replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(dist)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(Kst):
        graphs[i % ROTATE].replay()
    t1.record(stream)
    torch.cuda.synchronize()
    dist_barrier(dist)
    clk = clocks.stop()
    ms = dist_max(dist, t0.elapsed_time(t1), device) / Kst
    nv.nvfp4_check()
    bytes_step = M * K * 2
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    ach = bytes_step / (ms * 1e-3) / 1e9
    x0, g0, acc0 = sets[0]
    h_x = x0.cpu().pin_memory()
    h_m = torch.empty(8, dtype=torch.float64).pin_memory()

    def e2e_one():
        x0.copy_(h_x, non_blocking=True)
        graphs[0].replay()
        h_m.copy_(acc0["moments"], non_blocking=True)

    for _ in range(Wm):
        e2e_one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(Kst):
        e2e_one()
    b.record(stream)
    torch.cuda.synchronize()
    ms_e2e = dist_max(dist, a.elapsed_time(b) / Kst, device)  # max over ranks
    line = {
        "metric": METRIC, "value": bytes_step * world / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": world,
        "steps": Kst, "warmup": Wm, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 in, fp64/fp32 accumulation", "data": "synthetic (GDN prefill activation)",
        "config": {"workload": "activation_stats_32768x5120", "M": M, "K": K,
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": f"{ROTATE} rotating inputs, working set above the 126 MB L2"},
        "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                     "traffic": TRAFFIC_BYTES.get("actstats"), "peak_source": f"{peak_src} copy bandwidth",
                     "kernel": "nvfp4 activation stats", "ms_per_launch": ms},
        "clocks": clk,
        "e2e": {"value": bytes_step * world / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": bytes_step,
                "d2h_bytes_per_step": 64, "ms_per_step": ms_e2e},
        "gpu_launches": Kst,
        "summary": nv.activation_summary(acc0),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import nvfp4_oracle as o
        rows = 512
        g_np = np.float32(g0.item())
        t = time.perf_counter()
        n = 0
        while time.perf_counter() - t < args.cpu_seconds / 2 or n == 0:
            o.activation_stats(x_np[:rows], g_np)
            n += 1
        per = (time.perf_counter() - t) / n
        line["cpu_baseline"] = {"value": rows * K * 2 / per / 1e9, "unit": "GB/s", "cores": _blas_threads(),
                                "kind": "oracle", "sample": f"{rows} rows x {K} per pass ({n} passes)",
                                "host_cpus": os.cpu_count()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    for gr in graphs:
        del gr
    if dist is not None:
        dist.destroy_process_group()


GDN_REC_TOKENS = 32768  # the GDN projection's prefill length


def gdnrec_alg_bytes(T, H, H_k=None):
    """Bytes the delta-rule recurrence must move: q and k (BF16, 64 per head),
    v (BF16, 128 per head), beta and g (FP32), the BF16 output and the final
    FP32 state."""
    H_k = H if H_k is None else H_k
    per_token = 2 * (2 * H_k * 64) + 2 * H * 128 + 2 * 4 * H + 2 * H * 128
    return T * per_token + H * 128 * 64 * 4


def gdnrec_tensor_macs(T, H):
    """MACs the chunked kernels issue per step (TF32 m16n8k8 MMAs, 1024 MACs each):
    2016 per (chunk, head) in the per-chunk pass and 1024 in the state pass."""
    return -(-T // 64) * H * (2016 + 1024) * 1024


def run_gdnrec(args):
    """Delta-rule recurrence over the fused GDN projection's outputs at
    long-context prefill: q, k [32768, 32 x 64], v [32768, 32 x 128] BF16,
    beta and g [32768, 32] FP32, as the projection's epilogue writes them (one
    untimed layer call produces them); one nvfp4_gdn_recurrence call per step
    (two launches), BF16 output and the final state.  Inputs (545 MB) are
    larger than L2."""
    import torch
    from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
    from bit_quantized_linear_nvfp4_b200 import workloads as wl
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = dist_init(world)
    peaks, peak_src = load_peaks()
    w = wl.GDN
    T, H = GDN_REC_TOKENS, wl.GDN_HEADS
    proj = ProductStep("gdn", device)
    s0 = proj.sets[0]
    proj.linear(s0)
    torch.cuda.synchronize()
    q, k, v, _, beta, g = s0["outs"]
    for extra in proj.sets[1:]:
        extra.clear()
    proj.sets = [s0]
    if args.rows is not None:  # the first rows only: a smaller case of the same kernels (profiling)
        T = args.rows
        q, k, v, beta, g = (t[:T] for t in (q, k, v, beta, g))
    out = torch.empty((T, H * 128), dtype=torch.bfloat16, device=device)
    h_out = torch.empty((H, 128, 64), dtype=torch.float32, device=device)
    ws = torch.empty(nv.nvfp4_gdn_workspace_bytes(T, H), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def call():
        nv.nvfp4_gdn_recurrence(q, k, v, beta, g, out=out, h_out=h_out, workspace=ws)

    call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    Kst, Wm = args.steps, args.warmup
    for _ in range(Wm):
        graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(dist)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(Kst):
        graph.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    dist_barrier(dist)
    clk = clocks.stop()
    ms = dist_max(dist, t0.elapsed_time(t1), device) / Kst
    nv.nvfp4_check()
    bytes_step = gdnrec_alg_bytes(T, H)
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    ach = bytes_step / (ms * 1e-3) / 1e9
    macs = gdnrec_tensor_macs(T, H)
    tf32_peak = float(peaks["bf16_tflops_sustained"]) / 2.0
    # end to end: q, k, v, beta, g from pinned host memory, output and state back
    h_in = [t.cpu().pin_memory() for t in (q, k, v, beta, g)]
    h_res = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (out, h_out)]

    def e2e_one():
        for d, hh in zip((q, k, v, beta, g), h_in):
            d.copy_(hh, non_blocking=True)
        graph.replay()
        for hh, d in zip(h_res, (out, h_out)):
            hh.copy_(d, non_blocking=True)

    for _ in range(Wm):
        e2e_one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(Kst):
        e2e_one()
    b.record(stream)
    torch.cuda.synchronize()
    ms_e2e = dist_max(dist, a.elapsed_time(b) / Kst, device)  # max over ranks
    line = {
        "metric": METRIC, "value": bytes_step * world / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": world,
        "steps": Kst, "warmup": Wm, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "tf32 products, f32 state (bf16 in/out)",
        "data": "synthetic (the GDN projection's outputs on seeded N(0,1) activations and N(0,0.02) weights)",
        "config": {"workload": f"gdn_recurrence_{T}x{H}h_dk64_dv128", "tokens": T, "heads": H, "d_k": 64,
                   "d_v": 128, "chunk": 64, "parallelism": "replicas" if world > 1 else "single",
                   "l2": "inputs (545 MB) larger than the 126 MB L2"},
        "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                     "traffic": TRAFFIC_BYTES.get("gdnrec"), "peak_source": f"{peak_src} copy bandwidth",
                     "kernel": "gdn recurrence (per-chunk pass + state pass)", "ms_per_launch": ms},
        "kernels": {"tensor_macs_per_step": macs, "tensor_tflops": 2 * macs / (ms * 1e-3) / 1e12,
                    "tf32_peak_tflops": tf32_peak, "workspace_bytes": ws.numel()},
        "clocks": clk,
        "e2e": {"value": bytes_step * world / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in h_in),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in h_res), "ms_per_step": ms_e2e},
        "gpu_launches": 2 * Kst,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = _gdnrec_oracle_baseline(args.cpu_seconds / 2)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if dist is not None:
        dist.destroy_process_group()


def _gdnrec_oracle_baseline(seconds, steps=None):
    """The oracle's token loop on a bounded sample: 4 heads x 2048 tokens of
    seeded inputs with the recurrence's shapes, per pass."""
    from bit_quantized_linear_nvfp4_b200 import workloads as wl
    from oracle import nvfp4_oracle as o
    T, H = 2048, 4
    q, k, v, beta, g = wl.make_recurrence_inputs(T, H, H, 3)
    args = (q.reshape(T, H, 64), k.reshape(T, H, 64), v.reshape(T, H, 128), beta, g)
    t = time.perf_counter()
    n = 0
    while (steps is None and (time.perf_counter() - t < seconds or n == 0)) or (steps is not None and n < steps):
        o.gdn_recurrence(*args)
        n += 1
    per = (time.perf_counter() - t) / n
    val = gdnrec_alg_bytes(T, H) / per / 1e9
    return {"value": val, "unit": "GB/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{H} heads x {T} tokens per pass ({n} passes, oracle token loop)", "ms_per_pass": per * 1e3,
            "host_cpus": os.cpu_count()}


REFERENCE_BUDGET_S = 60.0  # timed oracle work of one reference-arm run, at most


def _time_oracle(fn, steps, warmup, budget_s=REFERENCE_BUDGET_S):
    """Run the oracle step fn min(warmup, 3) times untimed, then up to `steps`
    timed times, stopping once budget_s seconds are spent so that the whole run
    ends within a few minutes.  Returns (seconds per step, steps timed)."""
    for _ in range(min(warmup, 3)):
        fn()
    t = time.perf_counter()
    n = 0
    while n < steps:
        fn()
        n += 1
        if time.perf_counter() - t > budget_s:
            break
    return (time.perf_counter() - t) / n, n


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    if args.workload == "gdnrec":
        for _ in range(min(args.warmup, 1)):
            _gdnrec_oracle_baseline(0.0, steps=1)
        n = max(1, min(args.steps, 20))
        cb = _gdnrec_oracle_baseline(0.0, steps=n)
        val = cb["value"]
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": world,
                          "steps": n, "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": cb["ms_per_pass"],
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                          "dtype": "f64 (oracle)", "data": "synthetic",
                          "config": {"workload": f"gdn_recurrence_{GDN_REC_TOKENS}x32h_dk64_dv128",
                                     "tokens": GDN_REC_TOKENS, "heads": 32},
                          "cpu_baseline": cb,
                          "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return
    if args.workload == "actstats":
        from bit_quantized_linear_nvfp4_b200 import workloads as wl
        from oracle import nvfp4_oracle as o
        rows = 256
        x = wl.make_x(wl.GDN, rows=rows)
        g = o.global_scale(x)
        per, n = _time_oracle(lambda: o.activation_stats(x, g), args.steps, args.warmup)
        val = rows * x.shape[1] * 2 / per / 1e9
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": world,
                          "steps": n, "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                          "dtype": "f64 (oracle)", "data": "synthetic",
                          "config": {"workload": "activation_stats_32768x5120", "M": 32768, "K": x.shape[1]},
                          "cpu_baseline": {"value": val, "unit": "GB/s", "cores": _blas_threads(), "kind": "oracle",
                                           "sample": f"{rows} rows x {x.shape[1]} per step (oracle statistics)"},
                          "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return
    if args.workload == "kvfp8":
        from oracle import nvfp4_oracle as o
        rng = np.random.default_rng(6)
        rows, C = 2048, 1024
        x = rng.standard_normal((rows, C)).astype(np.float32)
        s = np.float32(np.abs(x).max() / 448)
        per, n = _time_oracle(lambda: o.kv_fp8_quantize(x, s), args.steps, args.warmup)
        val = rows * C * 3 / per / 1e9
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": world,
                          "steps": n, "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                          "dtype": "f32 (oracle)", "data": "synthetic",
                          "config": {"workload": "kv_fp8_encode_2x32768x1024", "tokens": 32768, "cols": C},
                          "cpu_baseline": {"value": val, "unit": "GB/s", "cores": _blas_threads(), "kind": "oracle",
                                           "sample": f"{rows} rows x {C} per step (oracle KV encode)"},
                          "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return
    if args.workload == "requant":
        from bit_quantized_linear_nvfp4_b200 import workloads as wl
        from oracle import nvfp4_oracle as o
        w = wl.GDN
        rows = 256
        wq = [o.quantize(sg) for sg in wl.make_w_segments(w)]
        c_all = np.concatenate([c for c, _, _ in wq])[:rows]
        s_all = np.concatenate([sf for _, sf, _ in wq])[:rows]
        g_rows = np.repeat(np.array([g for _, _, g in wq], np.float32), [sg.width for sg in w.segments])[:rows]
        g_c = max(g for _, _, g in wq)
        per, n = _time_oracle(lambda: o.requantize(c_all, s_all, g_rows, g_c), args.steps, args.warmup)
        val = 2 * rows * w.K * 0.5625 / per / 1e9
        sample = f"{rows} rows x {w.K} of the GDN weight per step (oracle requantize)"
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": world,
                          "steps": n, "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                          "dtype": "f32 (oracle)", "data": "synthetic",
                          "config": {"workload": "requant_gdn_weight_12352x5120", "N": 12352, "K": w.K},
                          "cpu_baseline": {"value": val, "unit": "GB/s", "cores": _blas_threads(), "kind": "oracle",
                                           "sample": sample},
                          "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return
    w, x, wq, g_a, extra = _prepare_oracle(args.workload)
    K = x.shape[1]
    rows = 16
    per, n = _time_oracle(lambda: _oracle_sample_step(args.workload, rows, x, wq, g_a, extra), args.steps,
                          args.warmup)
    if w is not None:
        val, unit = 2.0 * rows * w.N * K / per / 1e12, "TFLOP/s"
        cfg = {"workload": w.name, "M": w.M, "N": w.N, "K": w.K}
    else:
        val, unit = rows * K * 4.5625 / per / 1e9, "GB/s"
        cfg = {"workload": "quant", "M": x.shape[0], "K": K}
    sample = f"{rows} rows of the workload per step (quantise + FP64 GEMM + epilogue)"
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": unit, "n_gpus": world,
            "steps": n, "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
            "config": cfg,
            "cpu_baseline": {"value": val, "unit": unit, "cores": _blas_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="gdn",
                    choices=["oproj", "mlp", "gdn", "tiny", "decode1", "decode8", "decode64", "quant", "requant",
                             "kvfp8", "actstats", "gdnrec"])
    ap.add_argument("--impl", default="product", choices=["product", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-quant-line", action="store_true",
                    help="projection workloads: skip the standalone quantiser measurement on X[32768,17408]")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--rows", type=int, default=None,
                    help="quant: quantise [rows, 17408]; oproj/mlp/gdn: the first rows tokens; gdnrec: the first rows "
                         "tokens (smaller cases for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "requant":
        run_requant(args)
    elif args.workload == "kvfp8":
        run_kvfp8(args)
    elif args.workload == "actstats":
        run_actstats(args)
    elif args.workload == "gdnrec":
        run_gdnrec(args)
    else:
        run_product(args)


if __name__ == "__main__":
    main()
