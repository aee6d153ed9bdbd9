"""Benchmark of the fused attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one full pass of the hot path (one attn_fwd launch; for the FP8
workload the three preparation launches plus attn_fwd_fp8; for the MXFP8 workload
the three attn_quantize_mxfp8 launches plus attn_fwd_mxfp8) over one batch of
synthetic inputs already resident in HBM. The default workload is the LLM
training shape B=4, H=32, N=4096, d=128, causal, bf16: its inputs (403 MB) are
larger than L2 (126 MB), so no L2 flush is needed between timed iterations.
Timing uses CUDA events on the launching stream, W warm-up steps, then exactly K
timed steps bracketed by a barrier and device synchronisation; for N > 1 each
rank runs its own replica of the workload (the (batch, head) units are fully
independent, so the job shards with no data-path collective: weak scaling) and
the time is the maximum over ranks.

`--impl reference` times the fp64 CPU oracle (the only other implementation that
exists for this path) on a bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

import workloads  # noqa: E402

METRIC = "attention fwd TFLOPS (BF16 / FP8 / MXFP8) and % of B200 tensor-core peak"
METRIC_BWD = "attention bwd TFLOPS (BF16, 2.5x forward FLOPs) and % of B200 tensor-core peak"
METRIC_W4A16 = "W4A16 GEMM TFLOPS (fp16 activations, int4 weights dequantised on the fly) and % of HBM roofline"
DEFAULT_WORKLOAD = "llm_train_causal"
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: at least 20 and enough for ~10 ms, so that several clock "
                         "samples fall inside the timed window)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(workloads.WORKLOADS) + sorted(workloads.GEMM_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--sustained-steps", type=int, default=None,
                    help="after the timed region, time this many more steps (0: skip; default: at least "
                         "500 and enough for ~300 ms) and report them as 'sustained': a long loop meets "
                         "the 1 kW power cap")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward pass (attn_bwd) of a BF16 workload instead of the forward")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size (small profiling captures only)")
    return ap.parse_args()


# ------------------------------------------------------------------ distributed plumbing
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def init_dist(backend, world):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value, world, device=None):
    """Maximum of a float over all ranks (plumbing for the timing contract)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def shard_seed(w, rank):
    """Each rank draws its own replica of the workload (different data, same shape)."""
    return w.seed + 7919 * rank


# ------------------------------------------------------------------ clocks
REASON_NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class ClockSampler:
    """Samples the SM clock, its maximum and the throttle reasons while the timed
    region runs. NVML is read directly every ~2 ms (read-only queries), so even a
    timed region of ~10 ms holds several samples; without NVML, nvidia-smi is
    polled every 50 ms instead. Sampling is running before the timed region
    starts (entry waits for the first sample), every sample carries its host
    time, and the summary keeps the samples taken between mark_start() and
    mark_end() (all samples if none fall inside).

    A sample is (host time, sm MHz, max sm MHz, set of active reason names)."""
    SMI_FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
                  "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
                  "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id, period_s=0.002):
        self.gpu_id = gpu_id
        self.period_s = period_s
        self.samples = []
        self.window = None
        self.source = None
        self._stop = threading.Event()
        self.proc = None
        self.thread = None

    # ---- NVML
    def _nvml_loop(self, pynvml, h):
        bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
        mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self._stop.is_set():
            try:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            except pynvml.NVMLError:
                break
            self.samples.append((time.time(), float(sm), float(mx), {n for n, b in bits.items() if r & b}))
            time.sleep(self.period_s)

    def _start_nvml(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            gid = str(self.gpu_id)
            h = (pynvml.nvmlDeviceGetHandleByUUID(gid) if gid.startswith("GPU-")
                 else pynvml.nvmlDeviceGetHandleByIndex(int(gid)))
        except Exception:
            return False
        self.source = "nvml"
        self.thread = threading.Thread(target=self._nvml_loop, args=(pynvml, h), daemon=True)
        self.thread.start()
        return True

    # ---- nvidia-smi fallback
    def _smi_read(self):
        for line in self.proc.stdout:
            smp = self.parse_smi_line(time.time(), line)
            if smp is not None:
                self.samples.append(smp)

    @classmethod
    def parse_smi_line(cls, t, line):
        parts = [p.strip() for p in line.strip().split(",")]
        if len(parts) != len(cls.SMI_FIELDS):
            return None
        try:
            sm, mx = float(parts[0]), float(parts[1])
        except ValueError:
            return None
        return (t, sm, mx, {n for n, v in zip(REASON_NAMES, parts[3:]) if v.lower() == "active"})

    def _start_smi(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), "--query-gpu=" + ",".join(self.SMI_FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return False
        self.source = "nvidia-smi"
        self.thread = threading.Thread(target=self._smi_read, daemon=True)
        self.thread.start()
        return True

    def __enter__(self):
        if self._start_nvml() or self._start_smi():
            t0 = time.time()
            while not self.samples and time.time() - t0 < 10.0:
                time.sleep(0.005)
        return self

    def mark_start(self):
        self.window = [time.time(), None]

    def mark_end(self):
        if self.window is not None:
            self.window[1] = time.time()

    def __exit__(self, *exc):
        time.sleep(0.01)
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        import statistics
        samples = list(self.samples)
        inside = samples
        if self.window is not None and self.window[1] is not None:
            inside = [x for x in samples if self.window[0] <= x[0] <= self.window[1]]
        window_only = bool(inside) and self.window is not None and self.window[1] is not None
        use = inside if inside else samples
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        reasons = set()
        for x in use:
            reasons |= x[3]
        return {"sm_mhz": statistics.median(x[1] for x in use), "sm_max_mhz": max(x[2] for x in use),
                "reasons": sorted(reasons), "samples": len(use), "timed_window_only": window_only,
                "source": self.source}


def gpu_smi_id(dev, local):
    """nvidia-smi identifier (UUID) of a torch device, falling back to its index."""
    import torch
    uid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", "") or "")
    if uid:
        return uid if uid.startswith("GPU-") else "GPU-" + uid
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    return vis.split(",")[local] if vis else str(local)


def sustained_bf16_peak():
    """(rate, source): the measured bf16 GEMM rate over seconds under the power cap,
    else the pool's earlier measurement of it (1.4 PFLOP/s at ~1.3 GHz under the
    1 kW cap)."""
    path = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            v = json.load(f).get("bf16_tflops_sustained")
        if v:
            return v, "measured"
    return 1400.0, "fallback"


def measured_peaks():
    path = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d.get("bf16_tflops"), d.get("hbm_gbs"), "measured"
    return 1590.0, 6650.0, "fallback"


# ------------------------------------------------------------------ our arm
def l2_copies(w):
    """Input sets the timed loop rotates through: enough that the working set is at
    least twice the L2, so every step reads its inputs from HBM (1 for the large
    workloads, whose one set already exceeds it)."""
    set_bytes = 2 * w.B * w.H * w.N * w.d * 4 + 4 * w.B * w.H * w.N   # Q, K, V, O (bf16) + LSE
    return max(1, -(-2 * L2_BYTES // set_bytes))


class Step:
    """One pass of the hot path over resident inputs; returns launches per step.
    BF16 workloads smaller than L2 rotate through l2_copies(w) copies of their
    inputs and outputs, one per step."""

    def __init__(self, lib, w, x, dev):
        import torch
        self.lib, self.w = lib, w
        self.dev = dev
        self.copies = 1 if (w.fp8 or w.mx) else l2_copies(w)
        self.sets = []
        for c in range(self.copies):
            qkv = [x[n].to(dev) if c == 0 else x[n].to(dev).clone() for n in ("q", "k", "v")]
            o = torch.empty((w.B, w.H, w.N, w.d), device=dev, dtype=torch.bfloat16)
            lse = torch.empty((w.B, w.H, w.N), device=dev, dtype=torch.float32)
            self.sets.append((*qkv, o, lse))
        self.i = 0
        self.q, self.k, self.v, self.o, self.lse = self.sets[0]
        if w.fp8:
            self.rot = x["rot"].to(dev)
            T = (w.N + 127) // 128
            self.codes = [torch.empty((w.B, w.H, w.N, w.d), device=dev, dtype=torch.uint8) for _ in range(3)]
            self.scales = [torch.empty((w.B, w.H, T), device=dev, dtype=torch.float32) for _ in range(3)]
        if w.mx:
            self.codes = [torch.empty((w.B, w.H, w.N, w.d), device=dev, dtype=torch.uint8) for _ in range(3)]
            self.sfs = [torch.empty((w.B, w.H, w.N, w.d // 32), device=dev, dtype=torch.uint8) for _ in range(3)]
        self.launches = 4 if (w.fp8 or w.mx) else 1
        # attn_fwd runs launches with fewer two-Q-tile units than SMs on the
        # one-tile kernel (attn_fwd1_sm100), the rest on the two-tile kernel
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        one_tile = w.B * w.H * ((w.N + 255) // 256) < sms
        self.attn_kernel = "attn_fwd1_sm100" if (w.mx or (one_tile and not w.fp8)) else "attn_fwd_sm100"
        self.kernels = (["fp8_rotate_quantize", "fp8_quantize", "attn_fwd_sm100"] if w.fp8
                        else ["mxfp8_quantize", "attn_fwd1_sm100"] if w.mx else [self.attn_kernel])

    def run_device(self, stream, mark=None):
        """Launches one step on `stream`; mark(kernel name), if given, is called
        after each launch (the timed loop records a CUDA event there)."""
        lib, w = self.lib, self.w
        s = stream.cuda_stream
        mark = mark or (lambda name: None)
        if w.mx:
            for src, c8, sf in zip((self.q, self.k, self.v), self.codes, self.sfs):
                st = lib.attn_quantize_mxfp8(src.data_ptr(), c8.data_ptr(), sf.data_ptr(), w.B, w.H, w.N, w.d, s)
                if st:
                    raise lib.AttnError(st, "attn_quantize_mxfp8")
                mark("mxfp8_quantize")
            st = lib.attn_fwd_mxfp8(*(c.data_ptr() for c in self.codes), *(f.data_ptr() for f in self.sfs),
                                    self.o.data_ptr(), self.lse.data_ptr(), w.B, w.H, w.N, w.d, w.scale,
                                    int(w.causal), s)
            if st:
                raise lib.AttnError(st, "attn_fwd_mxfp8")
            mark("attn_fwd1_sm100")
            return
        if not w.fp8:
            q, k, v, o, lse = self.sets[self.i]
            self.i = (self.i + 1) % self.copies
            st = lib.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                              w.B, w.H, w.N, w.d, w.scale, int(w.causal), lib.ATTN_BF16, s)
            if st:
                raise lib.AttnError(st, "attn_fwd")
            mark(self.attn_kernel)
            return
        for src, rot, c8, sc in zip((self.q, self.k, self.v), (self.rot, self.rot, None), self.codes, self.scales):
            st = lib.attn_quantize_fp8(src.data_ptr(), None if rot is None else rot.data_ptr(), c8.data_ptr(),
                                       sc.data_ptr(), w.B, w.H, w.N, w.d, s)
            if st:
                raise lib.AttnError(st, "attn_quantize_fp8")
            mark("fp8_rotate_quantize" if rot is not None else "fp8_quantize")
        st = lib.attn_fwd_fp8(*(c.data_ptr() for c in self.codes), *(c.data_ptr() for c in self.scales),
                              self.o.data_ptr(), self.lse.data_ptr(), w.B, w.H, w.N, w.d, w.scale,
                              int(w.causal), s)
        if st:
            raise lib.AttnError(st, "attn_fwd_fp8")
        mark("attn_fwd_sm100")


class BwdStep:
    """One backward pass (attn_bwd: D_i, dK/dV, dQ) over resident inputs: Q, K, V,
    dO and the forward's O and LSE (computed once, outside the timed region)."""

    def __init__(self, lib, w, x, dev):
        import torch
        self.lib, self.w, self.dev = lib, w, dev
        self.q, self.k, self.v = (x[n].to(dev) for n in ("q", "k", "v"))
        g = torch.Generator().manual_seed(w.seed + 1)
        self.dout = torch.randn((w.B, w.H, w.N, w.d), generator=g).to(torch.bfloat16).to(dev)
        self.o, self.lse = lib.forward(self.q, self.k, self.v, causal=w.causal)
        self.grads = [torch.empty_like(self.q) for _ in range(3)]
        self.ws_bytes = lib.attn_bwd_workspace_bytes(w.B, w.H, w.N, w.d)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.copies = 1
        self.launches = 3
        self.kernels = ["attn_bwd"]

    def run_device(self, stream, mark=None):
        lib, w = self.lib, self.w
        st = lib.attn_bwd(self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(), self.o.data_ptr(),
                          self.lse.data_ptr(), self.dout.data_ptr(), *(t.data_ptr() for t in self.grads),
                          self.ws.data_ptr(), self.ws_bytes, w.B, w.H, w.N, w.d, w.scale, int(w.causal),
                          stream.cuda_stream)
        if st:
            raise lib.AttnError(st, "attn_bwd")
        if mark:
            mark("attn_bwd")


def time_e2e_bwd(lib, w, step, dev, stream, steps):
    """The backward end to end through the public Python API: Q, K, V, O, LSE and
    dO copied in from pinned host memory, dQ, dK, dV read back, every step."""
    import torch
    src = {"q": step.q, "k": step.k, "v": step.v, "o": step.o, "lse": step.lse, "dout": step.dout}
    host = {n: t.cpu().pin_memory() for n, t in src.items()}
    dev_in = {n: torch.empty_like(t) for n, t in src.items()}
    outs_h = [torch.empty(step.q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    outs_d = [torch.empty_like(step.q) for _ in range(3)]

    def one():
        with torch.cuda.stream(stream):
            for n in src:
                dev_in[n].copy_(host[n], non_blocking=True)
            lib.backward(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["o"], dev_in["lse"], dev_in["dout"],
                         causal=w.causal, dq=outs_d[0], dk=outs_d[1], dv=outs_d[2], workspace=step.ws,
                         stream=stream)
            for h, d_ in zip(outs_h, outs_d):
                h.copy_(d_, non_blocking=True)

    one()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs_h)
    return e0.elapsed_time(e1) / steps, h2d, d2h


class GemmStep:
    """One split-K W4A16 GEMM launch (w4a16_gemm_splitk) over resident operands.
    One operand set of the decode workload (117 MB of packed weights, 120 MB in
    all) fits in the 126 MB L2, so the timed loop rotates through enough copies
    that the working set is at least twice the L2: every step streams its
    weights from HBM."""

    def __init__(self, lib, wl, dev, seed):
        import torch
        self.lib, self.wl = lib, wl
        x, qw, s, z = workloads.make_w4a16(wl.M, wl.N, wl.K, seed)
        self.host = (x, qw, s, z)
        self.copies = max(1, -(-2 * L2_BYTES // self.bytes()))
        first = [t.to(dev) for t in (x, qw, s, z)]
        self.sets = [[t if c == 0 else t.clone() for t in first] +
                     [torch.empty((wl.M, wl.N), dtype=torch.float16, device=dev)] for c in range(self.copies)]
        self.i = 0
        self.x, self.qw, self.s, self.z, self.y = self.sets[0]
        self.ws_bytes = lib.w4a16_gemm_splitk_workspace_bytes(wl.M, wl.N, wl.K)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)
        torch.cuda.synchronize(dev)
        self.launches = 1
        self.kernels = ["w4a16_gemm_sm100"]

    def bytes(self):
        wl = self.wl
        return (wl.K * wl.N // 2 + (wl.K // 128) * wl.N * 3 + wl.M * wl.K * 2 + wl.M * wl.N * 2)

    def run_device(self, stream, mark=None):
        wl, lib = self.wl, self.lib
        x, qw, s, z, y = self.sets[self.i]
        self.i = (self.i + 1) % self.copies
        st = lib.w4a16_gemm_splitk(x.data_ptr(), qw.data_ptr(), s.data_ptr(), z.data_ptr(), y.data_ptr(),
                                   self.ws.data_ptr(), self.ws_bytes, wl.M, wl.N, wl.K, stream.cuda_stream)
        if st:
            raise lib.AttnError(st, "w4a16_gemm_splitk")
        if mark:
            mark("w4a16_gemm_sm100")


def run_gemm(args, lib, dev, rank, world, local):
    """Bench line of a W4A16 GEMM workload (HBM roofline on the algorithmic bytes:
    packed weights, scales, zero points, X read once, Y written once)."""
    import torch
    wl = workloads.GEMM_WORKLOADS[args.workload]
    stream = torch.cuda.Stream(dev)
    step = GemmStep(lib, wl, dev, wl.seed + 7919 * rank)
    args.steps = loop_steps(args.steps, estimate_step_ms(step, stream, world, dev), 10.0, 20)
    with ClockSampler(gpu_smi_id(dev, local)) as clk:
        ms_rank, kern_ms = time_device(step, stream, args.steps, max(3, args.warmup), world, dev, clk)
    st = lib.attn_get_device_status(stream.cuda_stream)
    if st != lib.ATTN_OK:
        raise lib.AttnError(st, "device status")
    clocks = clk.summary()
    ms_step = max_over_ranks(ms_rank, world, dev) / args.steps
    tflops = wl.flops * world / (ms_step * 1e-3) / 1e12
    _, hbm, peak_src = measured_peaks()
    k_ms = kern_ms["w4a16_gemm_sm100"]
    nbytes = step.bytes()
    gbs = nbytes / (k_ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
            "traffic": traffic_per_launch(wl.name), "peak_source": f"{peak_src} copy bandwidth",
            "kernel": "w4a16_gemm_sm100",
            "algorithmic_bytes": nbytes, "kernel_ms": round(k_ms, 5)}
    e2e = None
    if not args.no_e2e:
        host = [t.pin_memory() for t in step.host]
        dev_t = [torch.empty_like(t, device=dev) for t in host]
        y_h = torch.empty((wl.M, wl.N), dtype=torch.float16).pin_memory()

        def one():
            with torch.cuda.stream(stream):
                for h, d_ in zip(host, dev_t):
                    d_.copy_(h, non_blocking=True)
                lib.w4a16_matmul(*dev_t, out=step.y, stream=stream)
                y_h.copy_(step.y, non_blocking=True)
        one()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            one()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, world, dev)
        e2e = {"value": round(wl.flops * world / (e_ms * 1e-3) / 1e12, 3), "unit": "TFLOPS",
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host),
               "d2h_bytes_per_step": y_h.numel() * 2, "ms_per_step": round(e_ms, 4)}
    cpu = cpu_baseline_gemm(wl) if rank == 0 and world == 1 else None
    mhz = clocks.get("sm_mhz")
    return {
        "metric": METRIC_W4A16, "value": round(tflops, 3), "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp16xint4", "data": "synthetic",
        "config": {"workload": wl.name, "M": wl.M, "N": wl.N, "K": wl.K, "group": 128,
                   "parallelism": f"replicas x{world}",
                   "l2": f"one operand set is smaller than L2: the timed loop rotates through {step.copies} copies",
                   "schedule": "split-K over two CTAs per SM (w4a16_gemm_splitk)"},
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps,
        "kernel_ms": {k: round(v, 5) for k, v in kern_ms.items()},
        "cycles_per_step": None if mhz is None else round(ms_step * 1e-3 * mhz * 1e6), "clocks": clocks}


def cpu_baseline_gemm(wl, budget_s=10.0):
    """The W4A16 oracle as it stands, on 512 of the N output columns."""
    from oracle.w4a16 import w4a16_gemm_fp64
    x, qw, s, z = workloads.make_w4a16(wl.M, 512, wl.K, 99)
    args = (x.numpy(), qw.numpy(), s.numpy(), z.numpy())
    t0 = time.perf_counter()
    w4a16_gemm_fp64(*args)
    one = time.perf_counter() - t0
    reps = max(1, int(budget_s / max(one, 1e-3)))
    t0 = time.perf_counter()
    for _ in range(reps):
        w4a16_gemm_fp64(*args)
    dt = (time.perf_counter() - t0) / reps
    return {"value": round(2.0 * wl.M * 512 * wl.K / dt / 1e12, 6), "unit": "TFLOPS", "cores": blas_threads(),
            "kind": "oracle", "sample": f"{wl.M} x 512 x {wl.K} (512 of {wl.N} columns), {reps} repetitions"}


def estimate_step_ms(step, stream, world, dev):
    """Mean device time of one step over a few launches (after a short warm-up),
    the maximum over ranks, so that every rank sizes its loops alike."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(3):
            step.run_device(stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(5):
        step.run_device(stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return max_over_ranks(e0.elapsed_time(e1) / 5, world, dev)


def loop_steps(given, est_ms, target_ms, minimum):
    """Steps of a timed loop: the caller's count, else enough for target_ms."""
    if given is not None:
        return given
    return max(minimum, int(math.ceil(target_ms / max(est_ms, 1e-4))))


def time_device(step, stream, steps, warmup, world, dev, clk=None):
    """Returns (ms for `steps` steps on this rank, {kernel: mean ms per launch}).
    Events are recorded on the launching stream before the loop and after every
    launch, so each kernel's time is the gap between its neighbouring events."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step.run_device(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    marks = []

    def mark(name):
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(stream)
        marks.append((name, ev))

    # a one-launch step needs no events between launches: its kernel time is the step time
    many = step.launches > 1
    if clk is not None:
        clk.mark_start()
    e0.record(stream)
    for _ in range(steps):
        step.run_device(stream, mark if many else None)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if clk is not None:
        clk.mark_end()
    barrier(world, dev)
    total = e0.elapsed_time(e1)
    if not many:
        return total, {step.kernels[0]: total / steps}
    per = {}
    prev = e0
    for name, ev in marks:
        per.setdefault(name, []).append(prev.elapsed_time(ev))
        prev = ev
    return total, {k: sum(v) / len(v) for k, v in per.items()}



def time_e2e(lib, w, x, dev, stream, steps):
    """Same metric end to end through the public Python API: pinned host inputs
    copied in, forward, O and LSE read back, every step inside the timed region.
    BF16 goes through forward_from_host (the host-to-host entry, which overlaps
    the copies of head groups with the kernels); FP8 / MXFP8 copy in, quantise,
    attend and copy out on one stream."""
    import torch
    host = {n: x[n].pin_memory() for n in ("q", "k", "v")}
    o_host = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16).pin_memory()
    l_host = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    dq = dk = dv = do = dl = None
    if w.fp8 or w.mx:
        dq, dk, dv = (torch.empty_like(host[n], device=dev) for n in ("q", "k", "v"))
        do = torch.empty((w.B, w.H, w.N, w.d), device=dev, dtype=torch.bfloat16)
        dl = torch.empty((w.B, w.H, w.N), device=dev, dtype=torch.float32)
    extra = {}
    if w.fp8:
        extra["rot"] = x["rot"].to(dev)

    def one():
        with torch.cuda.stream(stream):
            if not (w.fp8 or w.mx):
                lib.forward_from_host(host["q"], host["k"], host["v"], causal=w.causal, out=o_host, lse=l_host,
                                      device=dev)
                return
            dq.copy_(host["q"], non_blocking=True)
            dk.copy_(host["k"], non_blocking=True)
            dv.copy_(host["v"], non_blocking=True)
            if w.fp8:
                q8, qs = lib.quantize_fp8(dq, extra["rot"], stream=stream)
                k8, ks = lib.quantize_fp8(dk, extra["rot"], stream=stream)
                v8, vs = lib.quantize_fp8(dv, None, stream=stream)
                lib.forward_fp8(q8, k8, v8, qs, ks, vs, causal=w.causal, out=do, lse=dl, stream=stream)
            else:
                q8, qs = lib.quantize_mxfp8(dq, stream=stream)
                k8, ks = lib.quantize_mxfp8(dk, stream=stream)
                v8, vs = lib.quantize_mxfp8(dv, stream=stream)
                lib.forward_mxfp8(q8, k8, v8, qs, ks, vs, causal=w.causal, out=do, lse=dl, stream=stream)
            o_host.copy_(do, non_blocking=True)
            l_host.copy_(dl, non_blocking=True)

    one()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    h2d = sum(host[n].numel() * host[n].element_size() for n in ("q", "k", "v"))
    d2h = o_host.numel() * 2 + l_host.numel() * 4
    return e0.elapsed_time(e1) / steps, h2d, d2h


SMS = 148
# dense tensor-core FLOPs per SM per clock (a 128x128x16 bf16 MMA step in 64 cycles;
# E4M3 at twice that rate) and NVIDIA's datasheet dense peaks
FLOP_PER_CLK_SM = {"bf16": 8192, "fp8": 16384}
DATASHEET_TFLOPS = {"bf16": 2250.0, "fp8": 4500.0}


def hw_peak_tflops(dt, sm_mhz):
    """Dense tensor-core peak of all SMs at the sampled SM clock."""
    return None if sm_mhz is None else SMS * FLOP_PER_CLK_SM[dt] * sm_mhz * 1e6 / 1e12


def prep_bytes(w):
    """Algorithmic bytes of one FP8 preparation launch: bf16 read, one code byte
    written per element, one fp32 scale per 128-token tile."""
    T = (w.N + 127) // 128
    return w.B * w.H * w.N * w.d * 3 + 4 * w.B * w.H * T


def mx_prep_bytes(w):
    """Algorithmic bytes of one MXFP8 quantisation launch: bf16 read, one code byte
    and 1/32 scale byte written per element."""
    n = w.B * w.H * w.N * w.d
    return 2 * n + n + n // 32


def roofline(w, kern_ms, sm_mhz, workload, kernel="attn_fwd_sm100"):
    """Roofline object of the dominant kernel (the attention kernel), from its
    mean launch time measured with CUDA events in the timed loop. The MXFP8
    attention kernel's S products run at the E4M3 rate and its P V products at
    the 16-bit rate, so its denominator is the bf16 peak x 4/3 (the time the
    tensor pipe needs for both products at those rates)."""
    peak_bf16, hbm, peak_src = measured_peaks()
    dt = "fp8" if w.fp8 else "bf16"
    k_ms = kern_ms[kernel]
    if w.N < 1024 and not w.fp8:
        # small N (ViT shapes): arithmetic intensity below the ridge point, so the
        # roofline is HBM: algorithmic bytes = Q, K, V read once + O written (bf16) + LSE (fp32)
        bytes_launch = 2 * w.B * w.H * w.N * w.d * 4 + 4 * w.B * w.H * w.N
        gbs = bytes_launch / (k_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(gbs / hbm, 4), "traffic": traffic_per_launch(workload),
                "peak_source": f"{peak_src} copy bandwidth", "kernel": "attn_fwd_sm100",
                "algorithmic_bytes": bytes_launch, "kernel_ms": round(k_ms, 5)}
    achieved = w.flops / (k_ms * 1e-3) / 1e12
    ratio = 2.0 if w.fp8 else (4.0 / 3.0 if w.mx else 1.0)
    peak = round(peak_bf16 * ratio, 1)
    note = {2.0: " x2 (fp8 nominal ratio)", 1.0: ""}.get(ratio, " x4/3 (E4M3 S at 2x, f16 P V at 1x the bf16 rate)")
    roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": traffic_per_launch(workload),
            "peak_source": f"{peak_src} bf16 burst" + note,
            "kernel": kernel, "algorithmic_flops": w.flops, "kernel_ms": round(k_ms, 5),
            "datasheet_peak": round(DATASHEET_TFLOPS["bf16"] * ratio, 1),
            "frac_of_datasheet_peak": round(achieved / (DATASHEET_TFLOPS["bf16"] * ratio), 4)}
    hw = hw_peak_tflops("bf16", sm_mhz)
    if hw:
        hw *= ratio
        roof["hw_peak_at_sampled_clock"] = round(hw, 1)
        roof["frac_of_hw_peak_at_sampled_clock"] = round(achieved / hw, 4)
    sus, sus_src = sustained_bf16_peak()
    # a long timed loop meets the 1 kW power cap (see "clocks"); the sustained
    # GEMM rate is the same-conditions denominator
    sus = round(sus * ratio, 1)
    roof["frac_of_sustained_peak"] = round(achieved / sus, 4)
    roof["sustained_peak"] = sus
    roof["sustained_peak_source"] = f"{sus_src} bf16 sustained" + note
    if w.fp8:
        pb = prep_bytes(w)
        roof["prep"] = {name: {"ms": round(kern_ms[name], 5), "algorithmic_bytes": pb,
                               "gbs": round(pb / (kern_ms[name] * 1e-3) / 1e9, 1),
                               "frac_of_hbm": round(pb / (kern_ms[name] * 1e-3) / 1e9 / hbm, 4)}
                        for name in ("fp8_rotate_quantize", "fp8_quantize") if name in kern_ms}
    if w.mx and "mxfp8_quantize" in kern_ms:
        pb = mx_prep_bytes(w)
        ms = kern_ms["mxfp8_quantize"]
        roof["prep"] = {"mxfp8_quantize": {"ms": round(ms, 5), "algorithmic_bytes": pb,
                                           "gbs": round(pb / (ms * 1e-3) / 1e9, 1),
                                           "frac_of_hbm": round(pb / (ms * 1e-3) / 1e9 / hbm, 4)}}
    return roof


def roofline_bwd(w, kern_ms, sm_mhz):
    """Roofline of the backward pass as one unit (its three launches: D_i, dK/dV,
    dQ), algorithmic FLOPs 2.5x the forward's, against the bf16 tensor-core peak."""
    peak, _, peak_src = measured_peaks()
    k_ms = kern_ms["attn_bwd"]
    fl = 2.5 * w.flops
    achieved = fl / (k_ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": None, "peak_source": f"{peak_src} bf16 burst",
            "kernel": "attn_bwd (attn_bwd_rowdot + attn_bwd_dkdv + attn_bwd_dq)", "algorithmic_flops": fl,
            "kernel_ms": round(k_ms, 5), "datasheet_peak": DATASHEET_TFLOPS["bf16"],
            "frac_of_datasheet_peak": round(achieved / DATASHEET_TFLOPS["bf16"], 4)}
    hw = hw_peak_tflops("bf16", sm_mhz)
    if hw:
        roof["hw_peak_at_sampled_clock"] = round(hw, 1)
        roof["frac_of_hw_peak_at_sampled_clock"] = round(achieved / hw, 4)
    return roof


def fp8_gemm_burst_tflops(dev, n=8192, reps=10):
    """Measured dense E4M3 GEMM rate (library GEMM, torch._scaled_mm, n^3, best of
    `reps`), the FP8 counterpart of the measured bf16 burst peak."""
    import torch
    try:
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        one = torch.ones((), device=dev, dtype=torch.float32)
        best = float("inf")
        for _ in range(reps + 2):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize(dev)
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return round(2.0 * n ** 3 / (best * 1e-3) / 1e12, 1)
    except Exception:
        return None


def run_ours(args):
    import torch
    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist("nccl", world)
    import exact_attention_forward_11_b200 as lib
    lib.load()
    if args.workload in workloads.GEMM_WORKLOADS:
        line = run_gemm(args, lib, dev, rank, world, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    w = workloads.WORKLOADS[args.workload]
    if args.batch is not None:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch)
    x = workloads.make_qkv(w.B, w.H, w.N, w.d, shard_seed(w, rank), w.outliers)
    x = {"q": x[0], "k": x[1], "v": x[2]}
    if w.fp8:
        x["rot64"], x["rot"] = workloads.make_rotation(w.d, w.seed + 7919)
    stream = torch.cuda.Stream(dev)
    if args.bwd and (w.fp8 or w.mx):
        raise SystemExit("--bwd needs a BF16 workload")
    step = BwdStep(lib, w, x, dev) if args.bwd else Step(lib, w, x, dev)
    est_ms = estimate_step_ms(step, stream, world, dev)
    args.steps = loop_steps(args.steps, est_ms, 10.0, 20)
    sustained_steps = loop_steps(args.sustained_steps, est_ms, 300.0, 500)
    with ClockSampler(gpu_smi_id(dev, local)) as clk:
        ms_rank, kern_ms = time_device(step, stream, args.steps, max(3, args.warmup), world, dev, clk)
    st = lib.attn_get_device_status(stream.cuda_stream)
    if st != lib.ATTN_OK:
        raise lib.AttnError(st, "device status")
    clocks = clk.summary()
    ms_total = max_over_ranks(ms_rank, world, dev)
    ms_step = ms_total / args.steps
    # the backward's 5 products (S, dP, dV, dK, dQ) against the forward's 2: 2.5x
    flops_rank = w.flops * (2.5 if args.bwd else 1.0)
    tflops = flops_rank * world / (ms_step * 1e-3) / 1e12
    # the same step over a long loop, after the timed region (the timed region
    # above is the line's value; this is the regime of a long training job)
    sustained = None
    if sustained_steps > 0:
        with ClockSampler(gpu_smi_id(dev, local)) as clk_s:
            ms_s, _ = time_device(step, stream, sustained_steps, 0, world, dev, clk_s)
        st = lib.attn_get_device_status(stream.cuda_stream)
        if st != lib.ATTN_OK:
            raise lib.AttnError(st, "device status")
        ms_s = max_over_ranks(ms_s, world, dev) / sustained_steps
        tf_s = flops_rank * world / (ms_s * 1e-3) / 1e12
        clocks_s = clk_s.summary()
        sustained = {"steps": sustained_steps, "ms_per_step": round(ms_s, 5), "value": round(tf_s, 3),
                     "unit": "TFLOPS", "clocks": clocks_s,
                     "cycles_per_step": (None if clocks_s.get("sm_mhz") is None
                                         else round(ms_s * 1e-3 * clocks_s["sm_mhz"] * 1e6))}
        if not args.bwd and w.N < 1024 and not w.fp8:
            # HBM-bound shapes: the sustained fraction is of the copy bandwidth
            # (the pool measures no separate sustained copy rate)
            _, hbm, hbm_src = measured_peaks()
            gbs = (2 * w.B * w.H * w.N * w.d * 4 + 4 * w.B * w.H * w.N) / (ms_s * 1e-3) / 1e9
            sustained.update({"achieved_gbs": round(gbs, 1), "frac_of_hbm_peak": round(gbs / hbm, 4),
                              "hbm_peak_source": f"{hbm_src} copy bandwidth"})
        else:
            sus_peak, sus_src = sustained_bf16_peak()
            ratio = 2.0 if w.fp8 else (4.0 / 3.0 if w.mx else 1.0)
            sustained.update({"frac_of_sustained_peak": round(tf_s / world / (sus_peak * ratio), 4),
                              "sustained_peak_source": f"{sus_src} bf16 sustained" +
                                                       ("" if ratio == 1.0 else f" x{ratio:.3g}")})
    # e2e through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        if args.bwd:
            e2e_ms, h2d, d2h = time_e2e_bwd(lib, w, step, dev, stream, args.e2e_steps)
        else:
            e2e_ms, h2d, d2h = time_e2e(lib, w, x, dev, stream, args.e2e_steps)
        e2e_ms = max_over_ranks(e2e_ms, world, dev)
        e2e = {"value": round(flops_rank * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOPS",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)}
    dt = "fp8" if w.fp8 else "bf16"
    roof = (roofline_bwd(w, kern_ms, clocks.get("sm_mhz")) if args.bwd
            else roofline(w, kern_ms, clocks.get("sm_mhz"), args.workload, step.attn_kernel))
    if w.fp8:
        roof["measured_fp8_gemm_burst_tflops"] = fp8_gemm_burst_tflops(dev)
    cpu = None
    if rank == 0 and world == 1:
        budget = float(os.environ.get("ATTN_CPU_BASELINE_S", "15"))
        cpu = cpu_baseline_bwd(w, budget) if args.bwd else cpu_baseline(w, budget_s=budget)
    mhz = clocks.get("sm_mhz")
    line = {
        "metric": METRIC_BWD if args.bwd else METRIC, "value": round(tflops, 3), "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3" if w.fp8 else ("mxfp8_e4m3_e8m0" if w.mx else "bf16"), "data": "synthetic",
        "config": {"workload": w.name, "B": w.B * world, "B_per_gpu": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": w.causal, "flops_per_step_per_gpu": flops_rank,
                   "pass": "backward" if args.bwd else "forward",
                   "parallelism": f"replicas x{world} (independent (b,h) units, no collective)",
                   "l2": "inputs larger than L2 (no flush)" if step.copies == 1 else
                   f"inputs smaller than L2: the timed loop rotates through {step.copies} copies "
                   f"(working set >= 2x L2, no flush)"},
        # the step's throughput against the datasheet dense tensor-core peak of the step's type
        "pct_of_peak": round(100 * tflops / world / DATASHEET_TFLOPS[dt], 2),
        "pct_of_peak_basis": f"B200 datasheet dense {dt.upper()} {DATASHEET_TFLOPS[dt]:.0f} TFLOP/s",
        "pct_of_measured_peak": round(100 * tflops / world / (measured_peaks()[0] *
                                                              (2 if w.fp8 else (4 / 3 if w.mx else 1))), 2),
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "sustained": sustained,
        "gpu_launches": step.launches * args.steps,
        "kernel_ms": {k: round(v, 5) for k, v in kern_ms.items()},
        "cycles_per_step": None if mhz is None else round(ms_step * 1e-3 * mhz * 1e6),
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def traffic_per_launch(workload):
    """DRAM bytes per launch from the committed ncu summary, if one matches."""
    path = os.path.join(HERE, "profiles", "traffic.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f).get(workload)
    return None


# ------------------------------------------------------------------ CPU oracle baseline
def oracle_sample(w, rows_per_head, heads, seed):
    """A bounded sample of the workload for the fp64 oracle: `heads` heads and
    `rows_per_head` query rows each. Returns (callable, algorithmic FLOPs)."""
    import numpy as np
    import torch
    gen = torch.Generator().manual_seed(seed)
    H = heads
    q = torch.randn((H, w.N, w.d), generator=gen).to(torch.bfloat16).double().numpy()
    k = torch.randn((H, w.N, w.d), generator=gen).to(torch.bfloat16).double().numpy()
    v = torch.randn((H, w.N, w.d), generator=gen).to(torch.bfloat16).double().numpy()
    rows = sorted(set(torch.randint(0, w.N, (rows_per_head,), generator=gen).tolist()))
    if w.causal:
        fl = sum(4.0 * (i + 1) * w.d for i in rows) * H
    else:
        fl = 4.0 * w.N * w.d * len(rows) * H
    from oracle import attention_fp64

    if w.mx:
        # the MXFP8 oracle: quantise and dequantise the sampled heads, then attend
        from oracle.mxfp8 import mx_dequantize, mx_quantize

        def call():
            qd, kd, vd = (mx_dequantize(*mx_quantize(t)) for t in (q, k, v))
            return attention_fp64(qd, kd, vd, w.scale, w.causal, rows=rows)
        return call, fl, (f"{H} head(s) x {len(rows)} query rows of {w.name} (N={w.N}, d={w.d}), "
                          f"MXFP8 quantisation of the sampled heads included")

    def call():
        return attention_fp64(q, k, v, w.scale, w.causal, rows=rows)
    return call, fl, f"{H} head(s) x {len(rows)} query rows of {w.name} (N={w.N}, d={w.d})"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count()


def cpu_baseline(w, budget_s=15.0):
    """Times the oracle as it stands on the host cores, on a bounded sample."""
    rows = 256
    call, fl, desc = oracle_sample(w, rows, 1, 12345)
    t0 = time.perf_counter()
    call()
    one = time.perf_counter() - t0
    reps = max(1, int(budget_s / max(one, 1e-3)))
    t0 = time.perf_counter()
    for _ in range(reps):
        call()
    dt = (time.perf_counter() - t0) / reps
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOPS", "cores": blas_threads(), "kind": "oracle",
            "sample": desc + f", fp64 numpy, {reps} repetitions"}


def cpu_baseline_bwd(w, budget_s=15.0):
    """The backward oracle as it stands on the host cores, one head of the workload
    in full (its algorithmic FLOPs: 2.5x the head's forward FLOPs)."""
    import torch
    from oracle import attention_bwd_fp64
    gen = torch.Generator().manual_seed(777)
    q, k, v, do = (torch.randn((1, 1, w.N, w.d), generator=gen).to(torch.bfloat16).double().numpy()
                   for _ in range(4))
    fl = 2.5 * w.flops / (w.B * w.H)
    t0 = time.perf_counter()
    attention_bwd_fp64(q, k, v, do, w.scale, w.causal)
    one = time.perf_counter() - t0
    reps = max(1, int(budget_s / max(one, 1e-3)))
    t0 = time.perf_counter()
    for _ in range(reps):
        attention_bwd_fp64(q, k, v, do, w.scale, w.causal)
    dt = (time.perf_counter() - t0) / reps
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOPS", "cores": blas_threads(), "kind": "oracle",
            "sample": f"1 head of {w.name} in full (N={w.N}, d={w.d}), fp64 numpy backward, {reps} repetitions"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    if args.steps is None:
        args.steps = 20   # each step is a bounded oracle sample of a few seconds at most
    if args.workload in workloads.GEMM_WORKLOADS:
        # each step: the W4A16 oracle on 128 of the N output columns
        wl = workloads.GEMM_WORKLOADS[args.workload]
        from oracle.w4a16 import w4a16_gemm_fp64
        ops = [t.numpy() for t in workloads.make_w4a16(wl.M, 128, wl.K, 4321)]

        def call():
            return w4a16_gemm_fp64(*ops)
        fl, desc, metric = 2.0 * wl.M * 128 * wl.K, f"{wl.M} x 128 x {wl.K} of {wl.name}", METRIC_W4A16
        cfg = {"workload": wl.name, "M": wl.M, "N": wl.N, "K": wl.K}
    elif args.bwd:
        # each step: the backward oracle on one head of the workload, N capped at 1024 rows
        w = workloads.WORKLOADS[args.workload]
        from oracle import attention_bwd_fp64
        n = min(w.N, 1024)
        gen = __import__("torch").Generator().manual_seed(4321)
        ops = [__import__("torch").randn((1, 1, n, w.d), generator=gen).double().numpy() for _ in range(4)]

        def call():
            return attention_bwd_fp64(*ops, w.scale, w.causal)
        fl = 2.5 * 4.0 * n * n * w.d / (2 if w.causal else 1)
        desc, metric = f"1 head of {w.name} with N = {n}", METRIC_BWD
        cfg = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "pass": "backward"}
    else:
        w = workloads.WORKLOADS[args.workload]
        # each step: one head x 64 query rows of the workload (bounded so that
        # warm-up + K steps finish within minutes)
        call, fl, desc = oracle_sample(w, 64, 1, 4321)
        metric = METRIC
        cfg = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal}
    for _ in range(max(1, args.warmup)):
        call()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        call()
    dt = (time.perf_counter() - t0) / args.steps
    v = fl / dt / 1e12
    line = {"impl": "reference", "metric": metric, "value": round(v, 6), "unit": "TFLOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": round(v, 6), "unit": "TFLOPS", "cores": blas_threads(), "kind": "oracle",
                             "sample": desc + " per step"},
            "e2e": {"value": round(v, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
