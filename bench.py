#!/usr/bin/env python3
"""Benchmark of the blockwise-scaled FP8 linear-layer hot path on B200.

One step = one training pass of the four Llama-3.1-8B-like linear layers
(tokens M = 8192; qkv 4096->6144, o_proj 4096->4096, gate_up 4096->28672,
down 14336->4096) through the library:
  requant all four weights (one batched call, the per-step recalibration),
  then per layer: quantize X (row-wise + column-wise copy), fprop,
  quantize dY (row-wise + column-wise copy), dgrad, wgrad.
Metric: FP8 blockwise linear TFLOP/s (fprop+dgrad+wgrad FLOPs / step time).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
With N > 1 (launched by torchrun) every rank runs an independent replica
(the path has no exchange step); value = all ranks' FLOPs / max time.
`--impl reference` times the CPU oracle on a bounded sample of the same
workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "FP8 blockwise linear TFLOP/s (fprop+dgrad+wgrad) & % FP8 peak; quant GB/s"
WORKLOAD = "llama3.1-8b-like linear layers, M=8192 tokens, fprop+dgrad+wgrad + act/weight quant + per-step requant"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="fp8bw", choices=["fp8bw", "reference"])
    p.add_argument("--mode", default="fp32", choices=["fp32", "pow2"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--no-steady", action="store_true", help="skip the >= 1.5 s steady-state region")
    p.add_argument("--e2e-steps", type=int, default=5)
    p.add_argument("--case", default=None,
                   help="time one call only (for profiling): fprop|dgrad|wgrad|quant_x|quant_dy|attn|"
                        "requant|bf16_fprop|wgrad_acc|quant_delayed_dy|quant_delayed_x on --layer at "
                        "--tokens, requant_sweep (32 layers), decode (FP8 KV-cache decode attention), or "
                        "moe_fprop|moe_dgrad|moe_wgrad "
                        "on the MoE expert layer --layer gate_up|down")
    p.add_argument("--sweep", action="store_true",
                   help="time every call of the Llama-like and MoE layers, both scale modes (one JSON line each)")
    p.add_argument("--layer", default="gate_up", choices=[n for n, _, _ in workloads.LLAMA8B_LAYERS])
    p.add_argument("--tokens", type=int, default=workloads.LLAMA8B_TOKENS,
                   help="tokens of the --case layer (32768 = the packed long-sequence batch)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_burst": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_burst": 1590.0, "bf16_sustained": 1400.0, "src": "fallback"}


def gemm_traffic():
    """DRAM bytes per GEMM launch from profiles/k_gemm_fp8_traffic.json (an
    ncu capture, summarised by hand), or None if the kernel source changed
    since those counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "k_gemm_fp8_traffic.json")
    src = os.path.join(ROOT, "blockwise_scaled_fp8_fp8bw_b200", "csrc", "gemm.cu")
    try:
        with open(path) as f:
            d = json.load(f)
        have = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        return int(d["traffic_bytes_per_launch"]) if have == d["gemm_cu_sha256_16"] else None
    except (OSError, KeyError, ValueError):
        return None


# ------------------------------------------------------------ clocks ------
def pci_bus_id(dev_index: int) -> str:
    """PCI bus id of a CUDA device (CUDA_VISIBLE_DEVICES-proof handle for NVML
    and nvidia-smi, whose indices are not CUDA's)."""
    p = torch.cuda.get_device_properties(dev_index)
    return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"


class ClockSampler:
    """SM clock and clock-event reasons of one GPU, sampled in a background
    thread every 10 ms through NVML (read-only queries), or every 100 ms by
    nvidia-smi where NVML is unavailable.  Only the samples taken between
    begin() and end() (the timed region, on the host clock) are summarised."""
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, dev_index: int):
        self.dev_index = dev_index
        self.bus = pci_bus_id(dev_index)
        self.samples = []          # (host time, sm MHz, set of active reasons)
        self.max_mhz = None
        self.window = [None, None]
        self.kind = None
        self._stop = threading.Event()
        self.thread = None
        self.proc = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByPciBusId(self.bus)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            bits = dict(zip(self.NAMES, (pynvml.nvmlClocksEventReasonHwSlowdown,
                                         pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                                         pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                                         pynvml.nvmlClocksEventReasonSwPowerCap)))

            def poll():
                while not self._stop.is_set():
                    mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((time.perf_counter(), float(mhz),
                                         {n for n, b in bits.items() if r & b}))
                    self._stop.wait(0.01)
                pynvml.nvmlShutdown()

            self.kind = "nvml, 10 ms"
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:  # no NVML: nvidia-smi by bus id
            pass
        try:
            q = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                 "clocks_event_reasons.sw_power_cap")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.bus, f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)

            def read():
                for line in self.proc.stdout:
                    f = [x.strip() for x in line.split(",")]
                    try:
                        mhz, self.max_mhz = float(f[0]), float(f[1])
                    except (ValueError, IndexError):
                        continue
                    act = {n for n, v in zip(self.NAMES, f[2:6]) if v.lower() == "active"}
                    self.samples.append((time.perf_counter(), mhz, act))

            self.kind = "nvidia-smi, 100 ms"
            self.thread = threading.Thread(target=read, daemon=True)
            self.thread.start()
        except OSError:
            self.kind = None

    def begin(self):
        self.window[0] = time.perf_counter()

    def end(self):
        self.window[1] = time.perf_counter()

    def stop(self):
        if self.kind is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no NVML or nvidia-smi"]}
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.thread.join(timeout=2)
        t0, t1 = self.window
        inside = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
        if not inside and self.samples:  # region shorter than the interval: the last sample before its end
            before = [x for x in self.samples if t1 is None or x[0] <= t1]
            inside = before[-1:] or self.samples[:1]
        reasons = set()
        for x in inside:
            reasons |= x[2]
        mhz = [x[1] for x in inside]
        return {"sm_mhz": float(np.median(mhz)) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(mhz), "sampler": self.kind}


# ----------------------------------------------------------- workload -----
class Layer:
    def __init__(self, name, K, N, M, dev, seed=0):
        self.name, self.K, self.N, self.M = name, K, N, M
        X, W, dY = workloads.llama_layer(name, seed=seed, device=dev, M=M)
        self.X, self.W, self.dY = X, W, dY
        u8, f32 = torch.uint8, torch.float32
        e = lambda *s, dt=u8: torch.empty(s, dtype=dt, device=dev)  # noqa: E731
        self.qx, self.sx, self.qxc, self.sxc = e(M, K), e(K // 128, M, dt=f32), e(K, M), e(M // 128, K, dt=f32)
        self.qd, self.sd, self.qdc, self.sdc = e(M, N), e(N // 128, M, dt=f32), e(N, M), e(M // 128, N, dt=f32)
        self.qw, self.sw, self.qwT = e(N, K), e(N // 128, K // 128, dt=f32), e(K, N)
        bf = torch.bfloat16
        self.Y, self.dX, self.dW = e(M, N, dt=bf), e(M, K, dt=bf), e(N, K, dt=bf)

    @property
    def flops(self):
        return 3 * 2 * self.M * self.N * self.K

    def act_bytes(self, rows, cols):
        # read bf16 + row codes + col codes + two fp32 scale grids
        return rows * cols * (2 + 1 + 1) + 2 * 4 * rows * cols // 128

    @property
    def weight_bytes(self):
        return self.N * self.K * (2 + 1 + 1) + 4 * self.N * self.K // (128 * 128)


def build_layers(dev, M=workloads.LLAMA8B_TOKENS):
    return [Layer(n, K, N, M, dev) for (n, K, N) in workloads.LLAMA8B_LAYERS]


def run_step(fb, layers, mode, ev=None):
    """One step.  If `ev` is a dict, CUDA events are recorded at the
    boundaries between calls of different kinds (one event ends a run of
    calls and starts the next, so a step carries 18 events for 21 launches);
    ev[kind] collects (start, end, launches) per run of consecutive calls of
    that kind."""
    calls = [("requant", lambda: fb.fp8bw_requant_weights([(l.W, l.qw, l.sw, l.qwT) for l in layers], mode))]
    for l in layers:
        calls += [
            ("quant_act", lambda l=l: fb.fp8bw_quant_act_1x128(l.X, mode, l.qx, l.sx, l.qxc, l.sxc)),
            ("gemm", lambda l=l: fb.fp8bw_gemm(fb.FP8BW_FPROP, l.qx, l.sx, l.qw, l.sw, l.Y, mode)),
            ("quant_act", lambda l=l: fb.fp8bw_quant_act_1x128(l.dY, mode, l.qd, l.sd, l.qdc, l.sdc)),
            ("gemm", lambda l=l: fb.fp8bw_gemm(fb.FP8BW_DGRAD, l.qd, l.sd, l.qwT, l.sw, l.dX, mode)),
            ("gemm", lambda l=l: fb.fp8bw_gemm(fb.FP8BW_WGRAD, l.qdc, l.sdc, l.qxc, l.sxc, l.dW, mode)),
        ]
    if ev is None:
        for _, fn in calls:
            fn()
        return

    def event():
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        return e

    start, n = event(), 0
    for i, (kind, fn) in enumerate(calls):
        fn()
        n += 1
        if i + 1 == len(calls) or calls[i + 1][0] != kind:
            end = event()
            ev.setdefault(kind, []).append((start, end, n))
            start, n = end, 0


LAUNCHES_PER_STEP = 1 + 4 * 5   # requant + per layer (2 quant_act + 3 gemm)


def bf16_ratio(fb, layers, reps=3):
    """Same three GEMMs per layer through the library's BF16 path."""
    dev = layers[0].X.device
    tot_flops, tot_ms = 0.0, 0.0
    for l in layers:
        WT = l.W.t().contiguous()
        dYT = l.dY.t().contiguous()
        XT = l.X.t().contiguous()
        D1 = torch.empty((l.M, l.N), dtype=torch.bfloat16, device=dev)
        D2 = torch.empty((l.M, l.K), dtype=torch.bfloat16, device=dev)
        D3 = torch.empty((l.N, l.K), dtype=torch.bfloat16, device=dev)
        calls = [lambda: fb.fp8bw_gemm_bf16(l.X, l.W, D1), lambda: fb.fp8bw_gemm_bf16(l.dY, WT, D2),
                 lambda: fb.fp8bw_gemm_bf16(dYT, XT, D3)]
        for c in calls:
            c()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(reps):
            for c in calls:
                c()
        e.record()
        torch.cuda.synchronize()
        tot_ms += s.elapsed_time(e) / reps
        tot_flops += l.flops
        del WT, dYT, XT, D1, D2, D3
    return tot_flops / (tot_ms * 1e-3) / 1e12


def attn_rates(fb, dev_index=0, reps=10):
    """FP8 attention forward over the packed 32K-token batch in both scale
    modes (outside the timed step): TFLOP/s of 10 launches after 3 warm-up,
    with the median SM clock sampled meanwhile (in the default run these
    launches follow seconds of GEMM load, so the clock is the power-capped
    one)."""
    out, mhz = {}, {}
    for name, mode in (("fp32", 0), ("pow2", 1)):
        fn, work, _ = attn_call(fb, mode=mode)
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ck = ClockSampler(dev_index)
        ck.start()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ck.begin()
        s.record()
        for _ in range(reps):
            fn()
        e.record()
        torch.cuda.synchronize()
        ck.end()
        mhz[name] = ck.stop()["sm_mhz"]
        out[name] = work / (s.elapsed_time(e) / reps * 1e-3) / 1e12
        del fn
        torch.cuda.empty_cache()
    out["sm_mhz"] = mhz
    out["workload"] = "packed 32768 tokens (4 sequences), 32 query / 8 KV heads of 128, causal"
    return out


def decode_rate(fb, hbm_gbs, reps=20):
    """FP8 KV-cache decode attention (outside the timed step): GB/s of the
    bytes one call reads and writes, 20 launches after 3 warm-up, against
    the copy bandwidth."""
    fn, work, _ = decode_call(fb)
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        fn()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / reps
    del fn
    torch.cuda.empty_cache()
    gbs = work / (ms * 1e-3) / 1e9
    return {"gbs": gbs, "frac_of_hbm": gbs / hbm_gbs, "ms": ms,
            "workload": "64 rollouts, 16K-token FP8 KV cache (lengths 762-16048), 32 query / 8 KV heads of 128"}


# ---------------------------------------------------------- CPU oracle ----
_ORC = {}


def _oracle_operands(name):
    """The oracle's quantized operands for a slice of one layer's fprop: the
    first 128 token rows of X and the first 512 rows of W (full K)."""
    if name not in _ORC:
        import oracle
        X, W, _ = workloads.llama_layer(name, seed=0, device="cpu", M=128)
        xb = X.view(torch.int16).numpy().view(np.uint16)
        wb = np.ascontiguousarray(W[:512].view(torch.int16).numpy().view(np.uint16))
        qx, sx, _, _ = oracle.quant_act_1x128(xb, 0, colwise=False)
        qw, sw, _ = oracle.quant_weight_128x128(wb, 0, transposed=False)
        _ORC[name] = (qx, sx, qw, sw)
    return _ORC[name]


def _oracle_gemm(name, rows, cols):
    import oracle
    qx, sx, qw, sw = _oracle_operands(name)
    t0 = time.perf_counter()
    oracle.gemm_ref_tile(0, qx, sx, qw, sw, 0, rows, 0, cols)
    dt = time.perf_counter() - t0
    return 2.0 * rows * cols * qx.shape[1], dt


def _cores():
    cores = len(os.sched_getaffinity(0))
    return min(cores, int(os.environ.get("OMP_NUM_THREADS", cores)))


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_quant_timing(name="qkv"):
    """The oracle's activation quantizer (1x128 row blocks + the column-wise
    copy) on one full tensor of the step, X of `name` at 8192 tokens, single
    threaded and on all host threads."""
    import oracle
    X, _, _ = workloads.llama_layer(name, seed=0, device="cpu")
    xb = X.view(torch.int16).numpy().view(np.uint16)
    M, K = xb.shape
    nbytes = M * K * (2 + 1 + 1) + 2 * 4 * M * K // 128
    out = {"tensor": f"X of {name} [{M},{K}] bf16, row blocks + column-wise copy, in full",
           "bytes": nbytes}
    allt = _cores()
    for label, n in (("single_thread", 1), ("all_threads", allt)):
        oracle.set_threads(n)
        t0 = time.perf_counter()
        oracle.quant_act_1x128(xb, 0)
        dt = time.perf_counter() - t0
        out[label] = {"threads": n, "s": dt, "GB/s": nbytes / dt / 1e9}
    oracle.set_threads(allt)
    return out


def oracle_sample(target_s=10.0, rows=8, cols=512):
    """Times the CPU oracle on the machine's host cores: its fp64 reference GEMM
    on a bounded sample of the step (blocks of `rows` x `cols` outputs of
    each layer's fprop, full K, cycling through the layers until about
    `target_s` seconds of GEMM work; `value`, extrapolated per FLOP), and its
    quantizer on one full tensor, single threaded and on all threads."""
    names = [n for n, _, _ in workloads.LLAMA8B_LAYERS]
    for n in names:
        _oracle_operands(n)
    flops = secs = 0.0
    i = 0
    while secs < target_s and i < 100000:
        n = names[i % len(names)]
        f, dt = _oracle_gemm(n, rows, cols)
        flops += f
        secs += dt
        i += 1
    quant = oracle_quant_timing()
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
            "cpu_model": cpu_model(), "nproc": os.cpu_count(),
            "sample": f"fp64 reference GEMM (oracle.gemm_ref_tile, fprop) on {i} blocks of "
                      f"{rows} rows x {cols} cols x full K cycling over the four layers "
                      f"({secs:.1f} s of CPU work), operands quantized by the oracle; "
                      "TFLOP/s = 2*rows*cols*K / time, extrapolated per FLOP to the step",
            "step_s_extrapolated": sum(l_flops for l_flops in
                                       [6 * workloads.LLAMA8B_TOKENS * N * K for _, K, N in workloads.LLAMA8B_LAYERS]
                                       ) / (flops / secs),
            "quant_act": quant}


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    names = [n for n, _, _ in workloads.LLAMA8B_LAYERS]
    for n in names:
        _oracle_operands(n)
    flops = secs = 0.0
    for i in range(args.warmup + args.steps):
        f, dt = _oracle_gemm(names[i % 4], 2, 256)
        if i >= args.warmup:
            flops += f
            secs += dt
    val = flops / secs / 1e12
    sample = ("one step = fp64 reference GEMM (oracle.gemm_ref_tile, fprop) of 2 rows x 256 "
              "cols x full K of one layer, cycling over the four layers")
    line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": secs * 1e3 / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD + " (CPU oracle, bounded sample)"},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------- one case -----
MOE_LAYERS = {"gate_up": (workloads.MOE_HIDDEN, 2 * workloads.MOE_INTER),
              "down": (workloads.MOE_INTER, workloads.MOE_HIDDEN)}


def moe_calls(fb, mode, layer):
    """Grouped GEMMs of one Qwen3-30B-A3B-like expert layer (128 experts,
    top-8 of 16384 tokens, Zipf(1.1) routing, segments padded to 128).
    FLOPs count the routed tokens (16384 * 8), not the padding rows."""
    dev = torch.device("cuda", 0)
    K, N = MOE_LAYERS[layer]
    r = workloads.moe_routing(0)
    G, Mt = len(r.counts), r.m_total_pad
    X = workloads.moe_permuted(r, K, 1.0, 11, dev)
    dY = workloads.moe_permuted(r, N, 1e-3, 12, dev)
    W = workloads.moe_experts(G, N, K, 13, dev)
    u8, f32, bf = torch.uint8, torch.float32, torch.bfloat16
    e = lambda *sh, dt=u8: torch.empty(sh, dtype=dt, device=dev)  # noqa: E731
    qx, sx, qxc, sxc = e(Mt, K), e(K // 128, Mt, dt=f32), e(K, Mt), e(Mt // 128, K, dt=f32)
    qd, sd, qdc, sdc = e(Mt, N), e(N // 128, Mt, dt=f32), e(N, Mt), e(Mt // 128, N, dt=f32)
    qw, sw, qwT = e(G, N, K), e(G, N // 128, K // 128, dt=f32), e(G, K, N)
    fb.fp8bw_quant_act_1x128(X, mode, qx, sx, qxc, sxc)
    fb.fp8bw_quant_act_1x128(dY, mode, qd, sd, qdc, sdc)
    fb.fp8bw_requant_weights([(W[g], qw[g], sw[g], qwT[g]) for g in range(G)], mode)
    off = torch.tensor(r.offsets, dtype=torch.int32, device=dev)
    Y, dX, dW = e(Mt, N, dt=bf), e(Mt, K, dt=bf), e(G, N, K, dt=bf)
    flops = 2 * workloads.MOE_TOKENS * workloads.MOE_TOPK * N * K
    return {
        "moe_fprop": (lambda: fb.fp8bw_grouped_gemm(fb.FP8BW_FPROP, off, qx, sx, qw, sw, Y, mode), flops, "TFLOP/s"),
        "moe_dgrad": (lambda: fb.fp8bw_grouped_gemm(fb.FP8BW_DGRAD, off, qd, sd, qwT, sw, dX, mode), flops, "TFLOP/s"),
        "moe_wgrad": (lambda: fb.fp8bw_grouped_gemm(fb.FP8BW_WGRAD, off, qdc, sdc, qxc, sxc, dW, mode), flops, "TFLOP/s"),
    }


def attn_call(fb, seed=0, mode=0):
    """FP8 attention forward over the packed long-sequence batch (32768
    tokens, 4 sequences), Llama-3.1-8B-like heads (32 query heads, 8 KV heads
    of 128), causal; Q, K, V quantized by the library's activation quantizer.
    FLOPs count the causal (query, key) pairs of the real tokens only:
    4 * 128 * Hq * sum_s n_s (n_s + 1) / 2 (Q.K^T and P.V)."""
    dev = torch.device("cuda", 0)
    T, Hq, Hkv, D = workloads.PACKED_TOKENS, 32, 8, 128
    off, ln = workloads.packed_segments(seed)
    Q = workloads.normal_bf16((T, Hq * D), 1.0, 31, dev)
    K = workloads.normal_bf16((T, Hkv * D), 1.0, 32, dev)
    V = workloads.normal_bf16((T, Hkv * D), 1.0, 33, dev)
    u8, f32 = torch.uint8, torch.float32
    e = lambda *sh, dt=u8: torch.empty(sh, dtype=dt, device=dev)  # noqa: E731
    q, sq, k, sk = e(T, Hq * D), e(Hq, T, dt=f32), e(T, Hkv * D), e(Hkv, T, dt=f32)
    vr, svr, vT, sv = e(T, Hkv * D), e(Hkv, T, dt=f32), e(Hkv * D, T), e(T // 128, Hkv * D, dt=f32)
    fb.fp8bw_quant_act_1x128(Q, mode, q, sq)
    fb.fp8bw_quant_act_1x128(K, mode, k, sk)
    fb.fp8bw_quant_act_1x128(V, mode, vr, svr, vT, sv)
    o = e(T, Hq * D, dt=torch.bfloat16)
    offd = torch.tensor(off, dtype=torch.int32, device=dev)
    lnd = torch.tensor(ln, dtype=torch.int32, device=dev)
    flops = 4 * D * Hq * sum(n * (n + 1) // 2 for n in ln)
    return (lambda: fb.fp8bw_attention_fwd(q, sq, k, sk, vT, sv, o, offd, lnd, 1, mode), flops, "TFLOP/s")


def decode_call(fb, seed=0, mode=0):
    """FP8 KV-cache decode attention: one new token for each of 64 rollouts
    over a 16K-token cache (the seeded length mix of workloads.decode_lengths),
    Llama-3.1-8B-like heads (32 query, 8 KV of 128); the cache quantized
    row-wise by the library's activation quantizer.  Work = the bytes the
    call must read or write: every cached token's K and V codes and scales
    (sum_b len_b * Hkv * 2 * (128 + 4)), the bf16 queries and outputs."""
    dev = torch.device("cuda", 0)
    lens, Lmax = workloads.decode_lengths(seed)
    B, Hq, Hkv, D = len(lens), 32, 8, 128
    T = B * Lmax
    u8, f32 = torch.uint8, torch.float32
    e = lambda *sh, dt=u8: torch.empty(sh, dtype=dt, device=dev)  # noqa: E731
    Q = workloads.normal_bf16((B, Hq * D), 1.0, 61, dev)
    k, sk, v, sv = e(T, Hkv * D), e(Hkv, T, dt=f32), e(T, Hkv * D), e(Hkv, T, dt=f32)
    X = workloads.normal_bf16((T, Hkv * D), 1.0, 62, dev)
    fb.fp8bw_quant_act_1x128(X, mode, k, sk)
    X = workloads.normal_bf16((T, Hkv * D), 1.0, 63, dev)
    fb.fp8bw_quant_act_1x128(X, mode, v, sv)
    del X
    torch.cuda.empty_cache()
    o = e(B, Hq * D, dt=torch.bfloat16)
    lnd = torch.tensor(lens, dtype=torch.int32, device=dev)
    nbytes = sum(lens) * Hkv * 2 * (D + 4) + 2 * B * Hq * D * 2
    return (lambda: fb.fp8bw_attention_decode(Q, k, sk, v, sv, o, lnd, Lmax), nbytes, "GB/s")


def run_case(args):
    """Times a single call of one layer (used for ncu captures and sweeps)."""
    import blockwise_scaled_fp8_fp8bw_b200 as fb
    torch.cuda.set_device(0)
    fb.fp8bw_init(0)
    mode = fb.FP8BW_SCALE_POW2 if args.mode == "pow2" else fb.FP8BW_SCALE_FP32
    name = args.layer
    if args.case.startswith("moe_"):
        fn, work, unit = moe_calls(fb, mode, name)[args.case]
        time_call(fb, args, name, mode, fn, work, unit)
        return
    if args.case == "attn":
        fn, work, unit = attn_call(fb, mode=mode)
        args.tokens = workloads.PACKED_TOKENS
        time_call(fb, args, "llama8b-packed-32k", mode, fn, work, unit)
        return
    if args.case == "decode":
        fn, work, unit = decode_call(fb, mode=mode)
        args.tokens = workloads.DECODE_BATCH
        time_call(fb, args, "llama8b-decode-64x16k", mode, fn, work, unit)
        return
    if args.case == "requant_sweep":
        # the per-step requant of 32 layers x 4 weights (about 7B parameters)
        dev = torch.device("cuda", 0)
        items, nbytes = [], 0
        for layer in range(32):
            for (n, K, N) in workloads.LLAMA8B_LAYERS:
                w = workloads.llama_weight(n, layer, device=dev)
                items.append((w, torch.empty((N, K), dtype=torch.uint8, device=dev),
                              torch.empty((N // 128, K // 128), dtype=torch.float32, device=dev),
                              torch.empty((K, N), dtype=torch.uint8, device=dev)))
                nbytes += N * K * 4 + 4 * (N // 128) * (K // 128)
        time_call(fb, args, "all", mode, lambda: fb.fp8bw_requant_weights(items, mode), nbytes, "GB/s")
        return
    calls = layer_calls(fb, mode, name, args.tokens, wgrad_acc=args.case == "wgrad_acc")
    fn, work, unit = calls[args.case]
    time_call(fb, args, name, mode, fn, work, unit)


def layer_calls(fb, mode, name, tokens, wgrad_acc=False):
    """Every timed call of one Llama-like layer at `tokens` tokens, with its
    algorithmic work (FLOP or bytes) and unit."""
    K, N = [(k, n) for nm, k, n in workloads.LLAMA8B_LAYERS if nm == name][0]
    l = Layer(name, K, N, tokens, torch.device("cuda", 0))
    fb.fp8bw_requant_weights([(l.W, l.qw, l.sw, l.qwT)], mode)
    fb.fp8bw_quant_act_1x128(l.X, mode, l.qx, l.sx, l.qxc, l.sxc)
    fb.fp8bw_quant_act_1x128(l.dY, mode, l.qd, l.sd, l.qdc, l.sdc)
    calls = {
        "fprop": (lambda: fb.fp8bw_gemm(fb.FP8BW_FPROP, l.qx, l.sx, l.qw, l.sw, l.Y, mode), l.flops / 3, "TFLOP/s"),
        "dgrad": (lambda: fb.fp8bw_gemm(fb.FP8BW_DGRAD, l.qd, l.sd, l.qwT, l.sw, l.dX, mode), l.flops / 3, "TFLOP/s"),
        "wgrad": (lambda: fb.fp8bw_gemm(fb.FP8BW_WGRAD, l.qdc, l.sdc, l.qxc, l.sxc, l.dW, mode), l.flops / 3, "TFLOP/s"),
        "quant_x": (lambda: fb.fp8bw_quant_act_1x128(l.X, mode, l.qx, l.sx, l.qxc, l.sxc), l.act_bytes(l.M, l.K), "GB/s"),
        "quant_dy": (lambda: fb.fp8bw_quant_act_1x128(l.dY, mode, l.qd, l.sd, l.qdc, l.sdc), l.act_bytes(l.M, l.N), "GB/s"),
        "requant": (lambda: fb.fp8bw_requant_weights([(l.W, l.qw, l.sw, l.qwT)], mode), l.weight_bytes, "GB/s"),
        "bf16_fprop": (lambda: fb.fp8bw_gemm_bf16(l.X, l.W, l.Y), l.flops / 3, "TFLOP/s"),
    }
    # per-tensor delayed scaling (history of 16, the comparison recipe):
    # dY in E5M2 and X in E4M3, each with its byte-transposed copy; 2 bytes
    # read and 2 written per element
    hist, sc, am = (torch.zeros(16, dtype=torch.float32, device=l.X.device),
                    torch.empty(1, dtype=torch.float32, device=l.X.device),
                    torch.empty(1, dtype=torch.float32, device=l.X.device))
    calls["quant_delayed_dy"] = (lambda: fb.fp8bw_quant_tensor_delayed(
        l.dY, fb.FP8BW_FMT_E5M2, mode, hist, l.qd, l.qdc, sc, am), 4 * l.M * l.N, "GB/s")
    calls["quant_delayed_x"] = (lambda: fb.fp8bw_quant_tensor_delayed(
        l.X, fb.FP8BW_FMT_E4M3, mode, hist, l.qx, l.qxc, sc, am), 4 * l.M * l.K, "GB/s")
    if wgrad_acc:   # wgrad added into an fp32 main gradient
        main_grad = torch.zeros((N, K), dtype=torch.float32, device=l.X.device)
        calls["wgrad_acc"] = (lambda: fb.fp8bw_gemm_f32(fb.FP8BW_WGRAD, l.qdc, l.sdc, l.qxc, l.sxc, main_grad,
                                                        accumulate=True, mode=mode), l.flops / 3, "TFLOP/s")
    return calls


SWEEP_CASES = ("fprop", "dgrad", "wgrad", "quant_x", "quant_dy", "requant")


def run_sweep(args):
    """Per-call table: every GEMM and quantizer call of the four Llama-like
    layers (at --tokens) and the two MoE expert layers, both scale modes, and
    the BF16 comparison GEMM, in one process; one JSON line per call."""
    import blockwise_scaled_fp8_fp8bw_b200 as fb
    torch.cuda.set_device(0)
    fb.fp8bw_init(0)
    for mname, mode in (("fp32", fb.FP8BW_SCALE_FP32), ("pow2", fb.FP8BW_SCALE_POW2)):
        args.mode = mname
        for name, _, _ in workloads.LLAMA8B_LAYERS:
            calls = layer_calls(fb, mode, name, args.tokens)
            for c in SWEEP_CASES + (("bf16_fprop",) if mname == "fp32" else ()):
                args.case = c
                fn, work, unit = calls[c]
                time_call(fb, args, name, mode, fn, work, unit)
            del calls
            torch.cuda.empty_cache()
        args.case = "attn"
        fn, work, unit = attn_call(fb, mode=mode)
        tokens, args.tokens = args.tokens, workloads.PACKED_TOKENS
        time_call(fb, args, "llama8b-packed-32k", mode, fn, work, unit)
        args.tokens = tokens
        del fn
        torch.cuda.empty_cache()
        args.case = "decode"
        fn, work, unit = decode_call(fb, mode=mode)
        tokens, args.tokens = args.tokens, workloads.DECODE_BATCH
        time_call(fb, args, "llama8b-decode-64x16k", mode, fn, work, unit)
        args.tokens = tokens
        del fn
        torch.cuda.empty_cache()
        for name in ("gate_up", "down"):
            mc = moe_calls(fb, mode, name)
            for c in ("moe_fprop", "moe_dgrad", "moe_wgrad"):
                args.case = c
                fn, work, unit = mc[c]
                time_call(fb, args, name, mode, fn, work, unit)
            del mc
            torch.cuda.empty_cache()


def time_call(fb, args, name, mode, fn, work, unit):
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.steps):
        fn()
    e.record()
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0
    ms = s.elapsed_time(e) / max(args.steps, 1)
    rate = work / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
    print(json.dumps({"case": args.case, "layer": name, "tokens": args.tokens, "mode": args.mode, "ms": ms,
                      unit: rate}), flush=True)


# ------------------------------------------------------------ ranks -------
def max_over_ranks(x: float, dist, device) -> float:
    """The job's time is its slowest rank's: the maximum of x over all ranks
    (x itself when there is one rank)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput of `world` replicas that each processed
    `units_per_rank` units, the slowest of them in `ms` milliseconds."""
    return units_per_rank * world / (ms * 1e-3)


# --------------------------------------------------------------- main -----
def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.case:
        run_case(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    def barrier():
        if dist:
            dist.barrier()

    from blockwise_scaled_fp8_fp8bw_b200 import build as _b
    if rank == 0 and not os.path.exists(os.path.join(ROOT, "blockwise_scaled_fp8_fp8bw_b200", "libfp8bw.so")):
        _b.build()
    barrier()
    import blockwise_scaled_fp8_fp8bw_b200 as fb
    fb.fp8bw_init(local)
    mode = fb.FP8BW_SCALE_POW2 if args.mode == "pow2" else fb.FP8BW_SCALE_FP32
    dev = torch.device("cuda", local)
    layers = build_layers(dev)
    torch.cuda.synchronize()

    for _ in range(max(args.warmup, 3)):
        run_step(fb, layers, mode)
    torch.cuda.synchronize()
    assert fb.fp8bw_last_device_error() == 0

    # ---- timed region: K steps, per-call events, clocks sampled meanwhile
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ev = {}
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks.begin()
    t0.record()
    for _ in range(args.steps):
        run_step(fb, layers, mode, ev)
    t1.record()
    torch.cuda.synchronize()
    clocks.end()
    barrier()
    ck = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    st = fb.fp8bw_last_device_error()
    if st != 0:
        raise RuntimeError(f"device error: {fb.status_string(st)}")
    ms_total = max_over_ranks(ms_total, dist, dev)
    ms_step = ms_total / args.steps
    step_flops = sum(l.flops for l in layers)
    value = job_rate(step_flops * args.steps, world, ms_total) / 1e12

    def kind_ms(k):
        return sum(s.elapsed_time(e) for s, e, _ in ev[k])

    gemm_ms = kind_ms("gemm") / (args.steps)
    quant_ms = kind_ms("quant_act") / args.steps
    req_ms = kind_ms("requant") / args.steps
    gemm_tflops = step_flops / (gemm_ms * 1e-3) / 1e12
    gemm_launch_ms = kind_ms("gemm") / sum(n for _, _, n in ev["gemm"])
    quant_bytes = sum(l.act_bytes(l.M, l.K) + l.act_bytes(l.M, l.N) for l in layers)
    req_bytes = sum(l.weight_bytes for l in layers)
    pk = peaks()
    # Half a second in, the step already runs at the power-capped clock
    # (median 1635 MHz over a 0.7 s region against 1965 max), so a region of
    # that length is rated against the sustained figure.
    timed_long = ms_total > 500.0
    fp8_peak = 2.0 * (pk["bf16_sustained"] if timed_long else pk["bf16_burst"])

    # ---- steady state: the same step timed for at least 1.5 s, so that the
    # clock has settled under the power cap (roofline against the sustained
    # BF16 figure)
    steady = None
    if not args.no_steady:
        n_steady = max(args.steps, int(np.ceil(1500.0 / ms_step)))
        ck2 = ClockSampler(local)
        ck2.start()
        time.sleep(0.3)
        ev2 = {}
        barrier()
        torch.cuda.synchronize()
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ck2.begin()
        q0.record()
        for _ in range(n_steady):
            run_step(fb, layers, mode, ev2)
        q1.record()
        torch.cuda.synchronize()
        ck2.end()
        barrier()
        ck2s = ck2.stop()
        q_ms = max_over_ranks(q0.elapsed_time(q1), dist, dev)
        st = fb.fp8bw_last_device_error()
        if st != 0:
            raise RuntimeError(f"device error (steady state): {fb.status_string(st)}")
        g2_ms = sum(a.elapsed_time(b) for a, b, _ in ev2["gemm"]) / n_steady
        g2_tflops = step_flops / (g2_ms * 1e-3) / 1e12
        steady = {"value": job_rate(step_flops * n_steady, world, q_ms) / 1e12, "unit": "TFLOP/s",
                  "ms_per_step": q_ms / n_steady, "steps": n_steady, "timed_s": q_ms / 1e3,
                  "gemm_tflops": g2_tflops, "gemm_peak": 2.0 * pk["bf16_sustained"],
                  "gemm_frac": g2_tflops / (2.0 * pk["bf16_sustained"]),
                  "peak_note": f"FP8 = 2 x {pk['src']} cuBLAS bf16 (sustained)", "clocks": ck2s}

    # ---- the same step with power-of-2 scales (block-scaled MMA path)
    pow2 = None
    if args.mode == "fp32":
        for _ in range(max(args.warmup, 3)):
            run_step(fb, layers, fb.FP8BW_SCALE_POW2)
        torch.cuda.synchronize()
        barrier()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record()
        for _ in range(args.steps):
            run_step(fb, layers, fb.FP8BW_SCALE_POW2)
        p1.record()
        torch.cuda.synchronize()
        p_ms = p0.elapsed_time(p1)
        p_ms = max_over_ranks(p_ms, dist, dev)
        st = fb.fp8bw_last_device_error()
        if st != 0:
            raise RuntimeError(f"device error (pow2): {fb.status_string(st)}")
        pow2 = {"value": job_rate(step_flops * args.steps, world, p_ms) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": p_ms / args.steps,
                "note": "same step with power-of-2 scales (GEMMs on the block-scaled MMA)"}

    # ---- BF16 comparison GEMMs (outside the timed region)
    bf16 = bf16_ratio(fb, layers) if rank == 0 else None
    attn = attn_rates(fb, local) if rank == 0 else None
    dec = decode_rate(fb, peaks()["hbm_gbs"]) if rank == 0 else None

    # ---- end to end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        host_in = [(l.X.cpu().pin_memory(), l.W.cpu().pin_memory(), l.dY.cpu().pin_memory()) for l in layers]
        host_out = [(torch.empty_like(l.Y, device="cpu").pin_memory(), torch.empty_like(l.dX, device="cpu").pin_memory(),
                     torch.empty_like(l.dW, device="cpu").pin_memory()) for l in layers]
        h2d = sum(x.numel() * 2 + w.numel() * 2 + d.numel() * 2 for x, w, d in host_in)
        d2h = sum(a.numel() * 2 + b.numel() * 2 + c.numel() * 2 for a, b, c in host_out)

        # Copies overlap the compute: host->device on one stream, device->host
        # on another, the layers in order on the compute stream.  The device
        # inputs and outputs are double-buffered across steps, so that step
        # k+1's uploads run while step k computes and step k's downloads run
        # while step k+1 computes.
        comp = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        bufs = [[(l.X, l.W, l.dY, l.Y, l.dX, l.dW) for l in layers],
                [tuple(torch.empty_like(t) for t in (l.X, l.W, l.dY, l.Y, l.dX, l.dW)) for l in layers]]
        in_free = [None, None]   # compute of the step that last read this input set is done
        out_free = [None, None]  # downloads of the step that last wrote this output set are done

        def e2e_step(k):
            b = k & 1
            dev_set = bufs[b]
            if in_free[b] is not None:
                s_in.wait_event(in_free[b])
            with torch.cuda.stream(s_in):
                for (x, w, d), (X, W, dY, _, _, _) in zip(host_in, dev_set):
                    W.copy_(w, non_blocking=True)
                ev_w = torch.cuda.Event()
                ev_w.record(s_in)
                ev_in = []
                for (x, w, d), (X, W, dY, _, _, _) in zip(host_in, dev_set):
                    X.copy_(x, non_blocking=True)
                    dY.copy_(d, non_blocking=True)
                    ev_in.append(torch.cuda.Event())
                    ev_in[-1].record(s_in)
            comp.wait_event(ev_w)
            fb.fp8bw_requant_weights([(W, l.qw, l.sw, l.qwT) for l, (_, W, _, _, _, _) in zip(layers, dev_set)],
                                     mode)
            if out_free[b] is not None:
                comp.wait_event(out_free[b])
            for i, (l, (X, W, dY, Y, dX, dW)) in enumerate(zip(layers, dev_set)):
                comp.wait_event(ev_in[i])
                fb.fp8bw_quant_act_1x128(X, mode, l.qx, l.sx, l.qxc, l.sxc)
                fb.fp8bw_gemm(fb.FP8BW_FPROP, l.qx, l.sx, l.qw, l.sw, Y, mode)
                fb.fp8bw_quant_act_1x128(dY, mode, l.qd, l.sd, l.qdc, l.sdc)
                fb.fp8bw_gemm(fb.FP8BW_DGRAD, l.qd, l.sd, l.qwT, l.sw, dX, mode)
                fb.fp8bw_gemm(fb.FP8BW_WGRAD, l.qdc, l.sdc, l.qxc, l.sxc, dW, mode)
                ev = torch.cuda.Event()
                ev.record(comp)
                s_out.wait_event(ev)
                with torch.cuda.stream(s_out):
                    a, bb, c = host_out[i]
                    a.copy_(Y, non_blocking=True)
                    bb.copy_(dX, non_blocking=True)
                    c.copy_(dW, non_blocking=True)
            in_free[b] = torch.cuda.Event()
            in_free[b].record(comp)
            out_free[b] = torch.cuda.Event()
            out_free[b].record(s_out)

        e2e_step(0)
        e2e_step(1)
        torch.cuda.synchronize()
        barrier()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        s_in.wait_stream(comp)
        for k in range(args.e2e_steps):
            e2e_step(k)
        comp.wait_stream(s_out)
        e.record()
        torch.cuda.synchronize()
        e_ms = s.elapsed_time(e)
        e_ms = max_over_ranks(e_ms, dist, dev)
        e2e = {"value": job_rate(step_flops * args.e2e_steps, world, e_ms) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e_ms / args.e2e_steps}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = oracle_sample(target_s=10.0)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens": workloads.LLAMA8B_TOKENS,
                       "layers": [f"{n}:{K}->{N}" for n, K, N in workloads.LLAMA8B_LAYERS],
                       "scale_mode": args.mode, "parallelism": f"replicas{world}",
                       "l2": "inputs larger than L2 (per-step working set > 1.5 GB)"},
            "roofline": {"bound": "tensor", "achieved": gemm_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": gemm_tflops / fp8_peak, "traffic": gemm_traffic(),
                         "kernel": "k_gemm_fp8 (all fprop/dgrad/wgrad launches)",
                         "peak_note": f"FP8 = 2 x {pk['src']} cuBLAS bf16 "
                                      f"({'sustained' if timed_long else 'burst'})",
                         "avg_launch_ms": gemm_launch_ms},
            "calls": {"gemm_ms_per_step": gemm_ms, "gemm_tflops": gemm_tflops,
                      "quant_act_ms_per_step": quant_ms, "quant_act_gbs": quant_bytes / (quant_ms * 1e-3) / 1e9,
                      "requant_ms_per_step": req_ms, "requant_gbs": req_bytes / (req_ms * 1e-3) / 1e9,
                      "hbm_peak_gbs": pk["hbm_gbs"],
                      "bf16_gemm_tflops": bf16, "fp8_over_bf16": (gemm_tflops / bf16) if bf16 else None,
                      "requant_over_step": req_ms / ms_step,
                      "attention_tflops": attn, "attention_decode": dec},
            "steady_state": steady,
            "pow2_scales": pow2,
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "gpu_launches_note": "library kernels in the timed region (K steps x 21); the steady-state, "
                                 "power-of-2 and e2e regions are timed separately",
            "clocks": ck,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
