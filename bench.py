"""Benchmark of the QLoRA NF4 hot path on B200.

A step is one pass of the whole path over the LLaMA-7B-shaped workload: for each of the three linear
shapes (N x K = 4096x4096, 11008x4096, 4096x11008) quantize the fp32 weight to NF4 with double-quantized
constants, dequantize it to bf16, and run the QLoRA linear forward (Y, U) and backward (dX, dA, dB) on
T = 16 x 512 tokens with LoRA r = 64, alpha = 16. Inputs are seeded synthetic tensors (see synth.py).

  value  linear fwd+bwd algorithmic TFLOP/s over the whole step (codec work inside the step time),
         summed over all ranks; inputs resident in HBM when the timed region starts
  e2e    the same through the public API with pinned host inputs: per step the H2D copy of every
         input (fp32 weights, X, dY, A, B) and the D2H read of the adapter gradients dA, dB; the
         copies run on their own stream, overlapping the kernels of the layer before
  roofline  the dominant kernel class (by measured share of device time), its algorithmic FLOP or
         bytes per launch over its mean CUDA-event duration, against MEASURED_PEAKS.json
  cpu_baseline  the oracle (fp64 numpy) on a 1/16 slice of the step, on this host's cores

Multi-GPU: the workload does not shard; every rank runs its own replica (weak scaling, no collective
on the data path), timed on the device and reduced with MAX over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s and NF4 dequant GB/s vs B200 roofline"
UNIT = "TFLOP/s"
SHAPES = [(4096, 4096), (11008, 4096), (4096, 11008)]
TOKENS, RANK_R, ALPHA = 16 * 512, 64, 16.0
SAMPLE_DIV = 16
WORKLOAD = ("LLaMA-7B-shaped QLoRA linears (N x K = 4096x4096, 11008x4096, 4096x11008), T = 16x512 tokens, "
            "r = 64, alpha = 16: quantize fp32 W to NF4 + double-quantized E4M3 constants, dequantize to "
            "bf16, linear forward and backward")
QUANT_B_PER_ELEM = 4 + 0.5 + 1 / 64 + 4 / 16384      # fp32 in; codes + E4M3 + fp32 scale2 out
DEQ_B_PER_ELEM = 0.5 + 1 / 64 + 4 / 16384 + 2        # stored NF4 in; bf16 out
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def fwd_flops(T, N, K, r):
    return 2 * T * N * K + 2 * T * r * (N + K)


def bwd_flops(T, N, K, r):
    return 2 * T * N * K + 4 * T * r * (N + K)


def step_flops(T=TOKENS, r=RANK_R):
    return sum(fwd_flops(T, N, K, r) + bwd_flops(T, N, K, r) for N, K in SHAPES)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---- distributed helpers (replicas; used with gloo in the CPU tests) ------------------------------

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---- clocks ---------------------------------------------------------------------------------------

class ClockSampler:
    """Samples the SM clock, its maximum, power and the active clock-event (throttle) reasons through
    NVML every few milliseconds on a background thread while the timed region runs (read-only queries;
    nothing about the GPU is changed)."""
    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, torch_device_index: int, period_s: float = 0.005):
        self.period, self.samples, self.stop_flag, self.thread, self.h = period_s, [], False, None, None
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
                self.h = nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.h = nv.nvmlDeviceGetHandleByIndex(torch_device_index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception:
            self.h = None

    def _run(self):
        nv = self.nv
        while not self.stop_flag:
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(self.h),
                                     nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.h is None:
            return
        import threading
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(timeout=5)
        if not self.samples:
            return None
        nv = self.nv
        reasons = sorted({name for _, bits, _ in self.samples for name, attr in self.REASONS.items()
                          if bits & getattr(nv, attr, 0)})
        return {"sm_mhz": statistics.median(s[0] for s in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples),
                "power_w_max": round(max(s[2] for s in self.samples), 1), "source": "NVML, 5 ms period"}


# ---- workload -------------------------------------------------------------------------------------

def make_workload(q, device, seed=0):
    import torch
    import synth
    wl = []
    for i, (N, K) in enumerate(SHAPES):
        c = synth.linear_case(TOKENS, N, K, RANK_R, ALPHA, seed=seed + 10 * i)
        d = dict(N=N, K=K)
        d["W"] = torch.from_numpy(c["W"]).to(device)
        for k in ("X", "A", "B", "dY"):
            d[k] = c[k].to(device)
        d["nf4"] = q.NF4Weight.empty(N, K, device)
        d["wsq"] = torch.empty(q.quantize_workspace_bytes(N * K), dtype=torch.uint8, device=device)
        d["deq"] = torch.empty(N, K, dtype=torch.bfloat16, device=device)
        d["wsl"] = torch.empty(q.linear_workspace_bytes(TOKENS, N, K, RANK_R), dtype=torch.uint8, device=device)
        d["Y"] = torch.empty(TOKENS, N, dtype=torch.bfloat16, device=device)
        d["U"] = torch.empty(TOKENS, RANK_R, dtype=torch.bfloat16, device=device)
        d["dX"] = torch.empty(TOKENS, K, dtype=torch.bfloat16, device=device)
        d["dA"] = torch.empty(RANK_R, K, dtype=torch.float32, device=device)
        d["dB"] = torch.empty(N, RANK_R, dtype=torch.float32, device=device)
        d["host"] = c
        wl.append(d)
    return wl


def run_layer(q, d, inp):
    """One layer of the step: outputs and workspaces from `d`, the five inputs from `inp`."""
    q.quantize(inp["W"], out=d["nf4"], workspace=d["wsq"])
    q.dequantize(d["nf4"], torch_bf16(), out=d["deq"])
    q.linear_fwd(inp["X"], d["nf4"], inp["A"], inp["B"], ALPHA, out=d["Y"], U_out=d["U"], workspace=d["wsl"])
    q.linear_bwd(inp["dY"], inp["X"], d["nf4"], inp["A"], inp["B"], ALPHA, U=d["U"], dX=d["dX"], dA=d["dA"],
                 dB=d["dB"], workspace=d["wsl"])


def run_step(q, wl):
    for d in wl:
        run_layer(q, d, d)


def torch_bf16():
    import torch
    return torch.bfloat16


# The headers each timed kernel class is compiled from (tile shapes, stage counts and CTA shapes are fixed
# there; the host sizes the persistent grids from the SM count alone); a DRAM-traffic record taken with ncu
# is used only while these files are unchanged.
KERNEL_SOURCES = {
    "fwd_gemm": ("common.cuh", "codec.cuh", "gemm_nf4w.cuh"),
    "bwd_gemm": ("common.cuh", "codec.cuh", "gemm_nf4w.cuh"),
    "quantize": ("common.cuh", "codec.cuh"),
    "dequantize": ("common.cuh", "codec.cuh"),
}


def source_hash(cls: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_nf4_quantized_14_b200", "csrc")
    for f in KERNEL_SOURCES[cls]:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(cls: str):
    """DRAM bytes per launch of a kernel class from the committed ncu summary, if it was taken on the
    class's current sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(cls)
    if not e or e.get("source_hash") != source_hash(cls):
        return None
    return e.get("bytes_per_launch")


def kernel_class(name: str):
    """(profiling class, label) of a kernel name as ncu prints it; the class is the library's timing class
    whose interval holds the launch (None for kernels outside the four measured classes)."""
    if "nf4_linear_gemm_kernel" in name:
        bwd = re.search(r"NF4WCfg<\s*(true|1)", name) is not None
        return ("bwd_gemm", "fused NF4 bwd (dX)") if bwd else ("fwd_gemm", "fused NF4 fwd (Y)")
    if "nf4_expand_scales_kernel" in name:
        by_col = re.search(r"nf4_expand_scales_kernel<\s*(true|1)", name) is not None
        return ("fwd_gemm", "constants by column (fwd)") if by_col else ("bwd_gemm", "constants by row (bwd)")
    for k in ("nf4_quantize_pass1", "nf4_mean", "nf4_dq_pass2"):
        if k in name:
            return "quantize", k
    if "nf4_dequantize_kernel" in name:
        return "dequantize", "nf4_dequantize_kernel"
    m = re.search(r"(\w+)(<[^(]*>)?\(", name.replace("void ", "").replace("qnf4::", ""))
    return None, (m.group(1) if m else name[:60])


def ncu_summary(csv_path: str, last: int, calls_per_class: int, command: str, out_path: str | None = None) -> int:
    """Per-kernel share of device time and DRAM bytes from an ncu launch list (metrics
    gpu__time_duration.sum, dram__bytes_read.sum, dram__bytes_write.sum; one pass per launch) over its last
    `last` launches, and profiles/traffic.json: DRAM bytes per timed call of each class (`calls_per_class`
    calls of each class in those launches)."""
    import csv
    rows = list(csv.reader(open(csv_path)))
    hi = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    hdr = rows[hi]
    ii, ki, mi, ui, vi = (hdr.index(c) for c in ("ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value"))
    scale = {"ns": 1e-3, "nsecond": 1e-3, "us": 1.0, "usecond": 1.0, "ms": 1e3, "msecond": 1e3, "byte": 1.0,
             "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    launches = {}
    for r in rows[hi + 1:]:
        if len(r) <= vi:
            continue
        d = launches.setdefault(int(r[ii]), {"name": r[ki]})
        d[r[mi]] = float(r[vi].replace(",", "")) * scale[r[ui]]
    sel = [launches[k] for k in sorted(launches)][-last:]
    agg, cls_bytes = {}, {}
    for d in sel:
        cls, label = kernel_class(d["name"])
        key = f"{label} [{cls}]" if cls else label
        a = agg.setdefault(key, [0, 0.0, 0.0, 0.0])
        rd, wr = d.get("dram__bytes_read.sum", 0.0), d.get("dram__bytes_write.sum", 0.0)
        a[0] += 1; a[1] += d.get("gpu__time_duration.sum", 0.0); a[2] += rd; a[3] += wr
        if cls:
            cls_bytes[cls] = cls_bytes.get(cls, 0.0) + rd + wr
    tot = sum(v[1] for v in agg.values())
    print(f"{len(sel)} launches, {tot:.1f} us total")
    print(f"{'share':>7} {'launches':>8} {'total us':>10} {'us/launch':>10} {'DRAM rd MB':>11} {'DRAM wr MB':>11}  kernel"
          "  (DRAM per launch)")
    for k, (n, t, rd, wr) in sorted(agg.items(), key=lambda x: -x[1][1]):
        print(f"{t / tot * 100:6.2f}% {n:8d} {t:10.1f} {t / n:10.1f} {rd / n / 1e6:11.1f} {wr / n / 1e6:11.1f}  {k}")
    out = {cls: {"bytes_per_launch": round(b / calls_per_class), "source_hash": source_hash(cls),
                 "calls": calls_per_class, "command": command} for cls, b in cls_bytes.items()}
    with open(out_path or os.path.join(ROOT, "profiles", "traffic.json"), "w") as f:
        json.dump(out, f, indent=1)
    for cls, e in out.items():
        print(f"# {cls}: {e['bytes_per_launch'] / 1e6:.1f} MB of DRAM traffic per timed call")
    return 0


def tensor_peak(peaks: dict, timed_s: float | None, clk: dict | None):
    """The bf16 denominator for a contraction timed inside the step: the burst figure (a short loop at
    full clock) when the timed region lasts under a second and the SM clock sampled during it sat at its
    maximum, otherwise the sustained figure (seconds of back-to-back GEMMs under the power cap)."""
    burst, sustained = peaks.get("bf16_tflops"), peaks.get("bf16_tflops_sustained")
    at_max = bool(clk and clk.get("sm_mhz") and clk.get("sm_max_mhz")
                  and clk["sm_mhz"] >= 0.97 * clk["sm_max_mhz"])
    if burst and (sustained is None or (timed_s is not None and timed_s < 1.0 and at_max)):
        why = (f"burst: timed region {timed_s:.3f} s < 1 s at SM clock {clk['sm_mhz']:.0f} of "
               f"{clk['sm_max_mhz']:.0f} MHz" if sustained else "burst (no sustained figure)")
        return burst, why
    why = ("sustained: " + (f"timed region {timed_s:.3f} s" if timed_s is not None else "timed region unknown")
           + (f", SM clock {clk['sm_mhz']:.0f} of {clk['sm_max_mhz']:.0f} MHz" if clk and clk.get("sm_mhz") else
              ", no clock samples"))
    return sustained, why


def roofline(prof: dict, steps: int, peaks: dict, peak_kind: str, timed_s: float | None = None,
             clk: dict | None = None):
    """Dominant kernel class by device time; its achieved rate against the measured peak. For a
    contraction the peak is the burst or the sustained bf16 figure (tensor_peak)."""
    per_step_units = {
        "fwd_gemm": sum(2 * TOKENS * N * K + 2 * TOKENS * RANK_R * N for N, K in SHAPES),
        "bwd_gemm": sum(2 * TOKENS * N * K + 2 * TOKENS * RANK_R * K for N, K in SHAPES),
        "quantize": sum(N * K for N, K in SHAPES) * QUANT_B_PER_ELEM,
        "dequantize": sum(N * K for N, K in SHAPES) * DEQ_B_PER_ELEM,
    }
    cls = max(per_step_units, key=lambda c: prof.get(c, (0, 0.0))[1])
    launches, ms = prof[cls]
    units_per_launch = per_step_units[cls] * steps / max(launches, 1)
    sec_per_launch = ms / 1e3 / max(launches, 1)
    if cls.endswith("gemm"):
        achieved = units_per_launch / sec_per_launch / 1e12
        peak, why = tensor_peak(peaks, timed_s, clk)
        out = {"bound": "tensor", "unit": "TFLOP/s", "kernel": cls}
        source = f"{peak_kind} bf16, {why}"
    else:
        achieved = units_per_launch / sec_per_launch / 1e9
        peak = peaks["hbm_gbs"]
        out = {"bound": "hbm", "unit": "GB/s", "kernel": cls}
        source = f"{peak_kind} (HBM copy)"
    out.update(achieved=round(achieved, 2), peak=peak, frac=round(achieved / peak, 4),
               traffic=traffic_for(cls), peak_source=source,
               launches=launches, mean_launch_us=round(sec_per_launch * 1e6, 2),
               algorithmic_per_launch=units_per_launch)
    return out


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_inputs(cases=None):
    """Host inputs of the oracle sample: for each shape, the first N/16 output features of the layer
    (weight rows, B rows, dY columns) with all T tokens. `cases` reuses already generated inputs."""
    import synth
    out = []
    for i, (N, K) in enumerate(SHAPES):
        c = cases[i] if cases is not None else synth.linear_case(TOKENS, N, K, RANK_R, ALPHA, seed=10 * i)
        n = N // SAMPLE_DIV
        out.append(dict(N=n, K=K, W=c["W"][:n].copy(), X=synth.bf16_values(c["X"]),
                        A=synth.bf16_values(c["A"]), B=synth.bf16_values(c["B"])[:n].copy(),
                        dY=synth.bf16_values(c["dY"])[:, :n].copy()))
    return out


def oracle_sample_flops():
    return sum(fwd_flops(TOKENS, N // SAMPLE_DIV, K, RANK_R) + bwd_flops(TOKENS, N // SAMPLE_DIV, K, RANK_R)
               for N, K in SHAPES)


def oracle_sample_step(inputs) -> float:
    """The oracle on 1/16 of a step: quantize + dequantize the first N/16 rows of each fp32 weight and
    run that narrower layer's forward and backward on all T tokens. Returns seconds."""
    import oracle as O
    t0 = time.perf_counter()
    for c in inputs:
        t = O.quantize(c["W"])
        Wt = O.bf16_bits_to_f32(O.dequantize(t, "bf16")).reshape(c["N"], c["K"])
        O.linear_fwd(c["X"], Wt, c["A"], c["B"], ALPHA)
        O.linear_bwd(c["dY"], c["X"], Wt, c["A"], c["B"], ALPHA)
    return time.perf_counter() - t0


SAMPLE_TEXT = (f"1/{SAMPLE_DIV} of a step: for each shape, the layer's first N/{SAMPLE_DIV} output features -- "
               f"quantize + dequantize those weight rows, then linear fwd + bwd of that narrower layer on all "
               f"{TOKENS} tokens")


def cpu_baseline_line(cases=None):
    inputs = oracle_inputs(cases)
    times = [oracle_sample_step(inputs) for _ in range(2)]
    sec = min(times)
    value = oracle_sample_flops() / sec / 1e12
    return {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{SAMPLE_TEXT}; best of {len(times)}; {sec:.2f} s per sample"}


# ---- arms -----------------------------------------------------------------------------------------

def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    inputs = oracle_inputs()
    for _ in range(args.warmup):
        oracle_sample_step(inputs)
    secs = [oracle_sample_step(inputs) for _ in range(args.steps)]
    sec = sum(secs) / len(secs)
    value = oracle_sample_flops() / sec / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": SAMPLE_TEXT},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                             "sample": f"{SAMPLE_TEXT}; {sec:.2f} s per sample"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_gpu(args):
    import torch
    import torch.distributed as dist
    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    import bit_nf4_quantized_14_b200 as q

    wl = make_workload(q, device)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        run_step(q, wl)
    torch.cuda.synchronize()
    if q.get_status() != 0:
        raise RuntimeError("device status set during warm-up")

    # ---- device-resident timing ----
    q.profile_read()
    q.profile_enable(True)
    clocks = ClockSampler(local_rank)
    barrier(device)
    torch.cuda.synchronize()
    clocks.start()
    n0 = q.kernel_launches()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        run_step(q, wl)
    ev1.record(stream)
    while not ev1.query():          # poll with sleeps so the sampler thread gets the interpreter
        time.sleep(0.0005)
    torch.cuda.synchronize()
    barrier(device)
    launches = q.kernel_launches() - n0
    clk = clocks.stop()
    q.profile_enable(False)
    prof = q.profile_read()
    status = q.get_status()
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, device)
    value = step_flops() * args.steps * world / (ms_max / 1e3) / 1e12

    # ---- end to end through the public API with pinned host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(q, wl, args, stream, device, world)
    secondary = None
    if rank == 0 and world == 1 and not args.no_secondary:
        secondary = secondary_figures(q, device)
    if rank == 0:
        emit(args, world, ms_max, value, e2e, launches, prof, clk, status, wl, secondary)
    if world > 1:
        barrier(device)
        dist.destroy_process_group()
    return 0


E2E_INPUTS = ("W", "X", "A", "B", "dY")


def run_e2e(q, wl, args, stream, device, world):
    """The step through the public API from pinned host buffers. Every step copies all five inputs of
    every layer host -> device and reads dA, dB back. The copies run on a stream of their own into two
    alternating sets of device input buffers: a layer's kernels wait on an event recorded after its
    copies, and a set is refilled only once the kernels that read it (two steps earlier) have finished,
    so the copies of the next layer and of the next step overlap the kernels of this one. The
    device -> host reads stay on the compute stream, behind the kernels that write dA and dB."""
    import torch
    host = []
    h2d = d2h = 0
    for d in wl:
        hb = {k: (torch.from_numpy(d["host"][k]) if k == "W" else d["host"][k]).pin_memory() for k in E2E_INPUTS}
        hb["dA"] = torch.empty_like(d["dA"], device="cpu").pin_memory()
        hb["dB"] = torch.empty_like(d["dB"], device="cpu").pin_memory()
        h2d += sum(hb[k].numel() * hb[k].element_size() for k in E2E_INPUTS)
        d2h += hb["dA"].numel() * 4 + hb["dB"].numel() * 4
        host.append(hb)
    sets = [[{k: d[k] for k in E2E_INPUTS} for d in wl],
            [{k: torch.empty_like(d[k]) for k in E2E_INPUTS} for d in wl]]
    copy = torch.cuda.Stream(device)
    free = [[None] * len(wl) for _ in sets]       # per set and layer: kernels done with its buffers
    nstep = [0]

    def e2e_step():
        s = nstep[0] & 1
        nstep[0] += 1
        ready = []
        with torch.cuda.stream(copy):
            for l, hb in enumerate(host):
                if free[s][l] is not None:
                    copy.wait_event(free[s][l])
                for k in E2E_INPUTS:
                    sets[s][l][k].copy_(hb[k], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy)
                ready.append(ev)
        for l, (d, hb) in enumerate(zip(wl, host)):
            stream.wait_event(ready[l])
            run_layer(q, d, sets[s][l])
            ev = torch.cuda.Event()
            ev.record(stream)
            free[s][l] = ev
            hb["dA"].copy_(d["dA"], non_blocking=True)
            hb["dB"].copy_(d["dB"], non_blocking=True)

    for _ in range(max(2, args.warmup // 2)):
        e2e_step()
    torch.cuda.synchronize()
    barrier(device)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy.wait_event(e0)             # no copy of the timed steps starts before the timed region
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)               # the compute stream waits on every copy, so e1 follows them all
    torch.cuda.synchronize()
    barrier(device)
    e_ms = max_over_ranks(e0.elapsed_time(e1), device)
    e2e_value = step_flops() * args.steps * world / (e_ms / 1e3) / 1e12
    return {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms / args.steps, 3),
            "copies": "host -> device on a copy stream into two alternating input sets, overlapping "
                      "the kernels; dA, dB read back on the compute stream"}


def emit(args, world, ms_max, value, e2e, launches, prof, clk, status, wl, secondary=None):
    peaks, kind = load_peaks()
    nq = sum(N * K for N, K in SHAPES) * args.steps
    parts = {}
    for c, (n, t) in prof.items():
        parts[c] = {"launches": n, "ms_total": round(t, 3)}
    if prof["quantize"][1] > 0:
        parts["quantize"]["GB/s"] = round(nq * QUANT_B_PER_ELEM / (prof["quantize"][1] / 1e3) / 1e9, 1)
    if prof["dequantize"][1] > 0:
        parts["dequantize"]["GB/s"] = round(nq * DEQ_B_PER_ELEM / (prof["dequantize"][1] / 1e3) / 1e9, 1)
    for c, f in (("fwd_gemm", lambda N, K: 2 * TOKENS * N * K + 2 * TOKENS * RANK_R * N),
                 ("bwd_gemm", lambda N, K: 2 * TOKENS * N * K + 2 * TOKENS * RANK_R * K)):
        if prof[c][1] > 0:
            parts[c]["TFLOP/s"] = round(sum(f(N, K) for N, K in SHAPES) * args.steps / (prof[c][1] / 1e3) / 1e12, 1)
    line = {"metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens": TOKENS, "r": RANK_R, "alpha": ALPHA,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "no flush: each step reads ~1.1 GB of distinct inputs (fp32 weights, X, dY), "
                             "well above the 126 MB L2"},
            "e2e": e2e,
            "gpu_launches": int(launches),
            "roofline": roofline(prof, args.steps, peaks, kind, timed_s=ms_max / 1e3, clk=clk),
            "clocks": clk, "parts": parts, "device_status": status}
    if secondary is not None:
        line["secondary"] = secondary
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_line([d["host"] for d in wl])
    print(json.dumps(line), flush=True)


# ---- secondary figures carried by the headline line -------------------------------------------------
# (the decode-shaped forward and one point of the codec sweep, so that the HBM-bound kernels are judged
# from the same run; the full sweeps stay under --workload decode | codec_sweep)

SECONDARY_DECODE = (22016, 8192, 1)          # N x K of a 65B gate/up projection, T = 1
SECONDARY_SWEEP_N = 1 << 28


def device_weight(N, K, gen, sigma=0.02, outlier_p=0.001):
    """N(0, sigma^2) with a fraction outlier_p of entries x10, drawn on the device (seeded)."""
    import torch
    W = torch.randn(N, K, device=gen.device, generator=gen).mul_(sigma)
    mask = torch.rand(N, K, device=gen.device, generator=gen) < outlier_p
    W[mask] *= 10.0
    return W


def device_sweep(n, gen, row=4096):
    """Sweep tensor: rows of `row` elements, sigma_row ~ U(0.005, 0.05), N(0, sigma_row^2), 0.1 % x10."""
    import torch
    rows = -(-n // row)
    sig = torch.empty(rows, 1, device=gen.device).uniform_(0.005, 0.05, generator=gen)
    x = (torch.randn(rows, row, device=gen.device, generator=gen) * sig).reshape(-1)[:n].contiguous()
    x[torch.rand(n, device=gen.device, generator=gen) < 0.001] *= 10.0
    return x


def secondary_figures(q, device, reps=20, warmup=3):
    import torch
    peaks, kind = load_peaks()
    gen = torch.Generator(device=device)
    gen.manual_seed(2026)
    flush = L2Flush(device)
    out = {"l2": L2_NOTE + "; median of %d calls, CUDA events" % reps,
           "peak": peaks["hbm_gbs"], "peak_source": f"{kind} (HBM copy)"}
    N, K, T = SECONDARY_DECODE
    W = device_weight(N, K, gen)
    nf4 = q.quantize(W)
    del W
    A = (torch.randn(RANK_R, K, device=device, generator=gen) * 0.01).to(torch.bfloat16)
    B = (torch.randn(N, RANK_R, device=device, generator=gen) * 0.01).to(torch.bfloat16)
    X = torch.randn(T, K, device=device, generator=gen).to(torch.bfloat16)
    Y = torch.empty(T, N, dtype=torch.bfloat16, device=device)
    U = torch.empty(T, RANK_R, dtype=torch.bfloat16, device=device)
    ws = torch.empty(q.linear_workspace_bytes(T, N, K, RANK_R), dtype=torch.uint8, device=device)
    n0 = q.kernel_launches()
    q.linear_fwd(X, nf4, A, B, ALPHA, out=Y, U_out=U, workspace=ws)
    launches = q.kernel_launches() - n0
    ms = time_calls(lambda: q.linear_fwd(X, nf4, A, B, ALPHA, out=Y, U_out=U, workspace=ws), flush, reps, warmup)
    ring = [nf4] + [nf4_copy(q, nf4) for _ in range(CHAIN_WEIGHTS - 1)]
    ms_chain = time_chain([lambda w=w: q.linear_fwd(X, w, A, B, ALPHA, out=Y, U_out=U, workspace=ws) for w in ring],
                          CHAIN_CALLS)
    byt = gemv_bytes(T, N, K, RANK_R)
    out["decode"] = {"workload": f"QLoRA linear forward, NF4 W {N} x {K}, T = {T}, r = {RANK_R}", "us": round(ms * 1e3, 2),
                     "bytes": int(byt), "GB/s": round(byt / (ms / 1e3) / 1e9, 1),
                     "frac": round(byt / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4), "launches_per_call": launches,
                     "chain": chain_entry(ms_chain, byt, peaks)}
    del nf4, ring, A, B, X, Y, U, ws
    n = SECONDARY_SWEEP_N
    x = device_sweep(n, gen).view(1, n)
    xb = x.to(torch.bfloat16)
    qn = q.NF4Weight.empty(1, n, device)
    wsq = torch.empty(q.quantize_workspace_bytes(n), dtype=torch.uint8, device=device)
    deq = torch.empty(1, n, dtype=torch.bfloat16, device=device)
    sweep = {"workload": f"sweep tensor of 2^{n.bit_length() - 1} elements (rows of 4096, sigma_row ~ "
                         f"U(0.005, 0.05), 0.1 % x10 outliers)"}
    for name, fn, bpe in (("quantize_fp32", lambda: q.quantize(x, out=qn, workspace=wsq), QUANT_B_PER_ELEM),
                          ("quantize_bf16", lambda: q.quantize(xb, out=qn, workspace=wsq), QUANT_B_PER_ELEM - 2),
                          ("dequantize_bf16", lambda: q.dequantize(qn, torch.bfloat16, out=deq), DEQ_B_PER_ELEM)):
        ms = time_calls(fn, flush, reps, warmup)
        sweep[name] = {"us": round(ms * 1e3, 2), "GB/s": round(n * bpe / (ms / 1e3) / 1e9, 1),
                       "frac": round(n * bpe / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4)}
    out["codec_2^28"] = sweep
    del x, xb, qn, wsq, deq, flush
    torch.cuda.empty_cache()
    return out


# ---- secondary workloads: decode-shaped forward and the codec sweep ------------------------------
# (python bench.py --workload decode | codec_sweep; one JSON line each, with every case listed)

DECODE_TOKENS = (1, 4, 16)
DECODE_WORKLOAD = ("LLaMA-65B-shaped frozen NF4 linears (N x K = 8192x8192, 22016x8192, 8192x22016), "
                   "forward only at T = 1, 4, 16 tokens, r = 64, alpha = 16")
SWEEP_SIZES = tuple(2 ** e for e in (20, 22, 24, 26, 28, 30, 31))


def gemv_bytes(T, N, K, r):
    """Algorithmic HBM bytes of one decode-shaped forward: the stored NF4 weight, A and B, X in, Y out."""
    return (0.5 + 1 / 64 + 4 / 16384) * N * K + 2 * r * (N + K) + 2 * T * (N + K)


CHAIN_WEIGHTS = 6     # distinct copies of the weight a chain cycles through (6 x 34 MB and more: > L2)
CHAIN_CALLS = 16


def nf4_copy(q, w):
    """A copy of an NF4 weight in new device memory (same values, distinct addresses)."""
    return q.NF4Weight(w.codes.clone(), w.absmax_e4m3.clone(), w.scale2.clone(), w.offset.clone(), w.rows, w.cols)


def chain_entry(ms, byt, peaks):
    return {"us": round(ms * 1e3, 2), "GB/s": round(byt / (ms / 1e3) / 1e9, 1),
            "frac": round(byt / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
            "how": f"{CHAIN_CALLS} calls back to back over {CHAIN_WEIGHTS} copies of the weight in distinct memory "
                   "(consecutive layers of a decode step), enqueued behind a device sleep; no flush"}


L2_NOTE = ("flushed before every timed call: a 512 MB write, then a read of another 512 MB buffer, so the "
           "timed call finds neither its inputs nor dirty lines in L2")


class L2Flush:
    """Evict what the next timed call reads from L2 and leave L2 clean. A 512 MB write (4x the 126 MB L2)
    evicts everything but leaves L2 full of dirty lines, which the timed call then pays to write back as
    it evicts them (for a 90 MB read, about a third more time; `--workload flush_check` measures it); a
    full read of a second 512 MB buffer afterwards replaces them with clean lines of that buffer."""

    def __init__(self, device):
        import torch
        self.w = torch.empty(512 << 20, dtype=torch.uint8, device=device)
        self.r = torch.zeros(64 << 20, dtype=torch.int64, device=device)
        self.i = 0

    def write_only(self):
        self.i += 1
        self.w.fill_(self.i & 0xFF)

    def __call__(self):
        self.write_only()
        self.r.sum()


def time_calls(fn, flush, reps, warmup=3):
    """Median device time (ms) of fn() over reps calls, the L2 flushed (flush()) before each, outside the
    timed pair of events, on the same stream."""
    import torch
    for _ in range(warmup):
        fn()
    stream = torch.cuda.current_stream()
    times = []
    for i in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.median(times)


def time_chain(fns, calls, reps=5):
    """Median per-call device time (ms) of `calls` calls enqueued back to back, cycling through fns (calls on
    distinct weights whose total exceeds L2, as the layers of a decode step do), behind a 1 ms device sleep
    so the host's enqueueing is not timed."""
    import torch
    for f in fns:
        f()
    stream = torch.cuda.current_stream()
    per = []
    for _ in range(reps):
        torch.cuda._sleep(2_000_000)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(calls):
            fns[i % len(fns)]()
        b.record(stream)
        b.synchronize()
        per.append(a.elapsed_time(b) / calls)
    return statistics.median(per)


def run_flush_check(args):
    """How the L2 flush before a timed call changes what it measures, on a plain torch read (a sum over
    90 MB and 34 MB, the sizes of the decode layers' NF4 weights): after a write-only flush, after the
    write-then-read flush the other measurement lines use, with no flush (inputs L2-resident), and as a
    chain over distinct copies. Library kernels only; none of this package's."""
    import torch
    device = torch.device("cuda", 0)
    flush = L2Flush(device)
    cases = []
    for mb in (90, 34):
        ring = [torch.ones((mb << 20) // 8, dtype=torch.int64, device=device) for _ in range(CHAIN_WEIGHTS)]
        fn = lambda: ring[0].sum()
        row = {"MB": mb}
        row["write_flush_us"] = round(time_calls(fn, flush.write_only, args.steps, args.warmup) * 1e3, 2)
        row["write_read_flush_us"] = round(time_calls(fn, flush, args.steps, args.warmup) * 1e3, 2)
        row["no_flush_us"] = round(time_calls(fn, lambda: None, args.steps, args.warmup) * 1e3, 2)
        row["chain_us"] = round(time_chain([lambda t=t: t.sum() for t in ring], CHAIN_CALLS) * 1e3, 2)
        cases.append(row)
        del ring
    print(json.dumps({"metric": "device time of a torch sum over a weight-sized tensor under each L2 preparation",
                      "unit": "us", "steps": args.steps, "warmup": args.warmup, "cases": cases}), flush=True)
    return 0


def run_decode(args):
    import torch
    import synth
    import bit_nf4_quantized_14_b200 as q
    peaks, kind = load_peaks()
    device = torch.device("cuda", 0)
    flush = L2Flush(device)
    cases = []
    for i, (N, K) in enumerate(synth.LLAMA65B_SHAPES):
        W = torch.from_numpy(synth.weight_f32(N, K, seed=40 + i, tensor_id=1)).to(device)
        nf4 = q.quantize(W)
        del W
        ring = [nf4] + [nf4_copy(q, nf4) for _ in range(CHAIN_WEIGHTS - 1)]
        A = synth.to_bf16(synth.normal_f32((RANK_R, K), 0.01, 40 + i, 3)).to(device)
        B = synth.to_bf16(synth.normal_f32((N, RANK_R), 0.01, 40 + i, 4)).to(device)
        X16 = synth.to_bf16(synth.normal_f32((max(DECODE_TOKENS), K), 1.0, 40 + i, 2)).to(device)
        for T in DECODE_TOKENS:
            X = X16[:T].contiguous()
            Y = torch.empty(T, N, dtype=torch.bfloat16, device=device)
            U = torch.empty(T, RANK_R, dtype=torch.bfloat16, device=device)
            ws = torch.empty(q.linear_workspace_bytes(T, N, K, RANK_R), dtype=torch.uint8, device=device)
            fn = lambda: q.linear_fwd(X, nf4, A, B, ALPHA, out=Y, U_out=U, workspace=ws)
            n0 = q.kernel_launches()
            fn()
            launches = q.kernel_launches() - n0
            ms = time_calls(fn, flush, args.steps, args.warmup)
            ms_chain = time_chain([lambda w=w: q.linear_fwd(X, w, A, B, ALPHA, out=Y, U_out=U, workspace=ws)
                                   for w in ring], CHAIN_CALLS)
            gbs = gemv_bytes(T, N, K, RANK_R) / (ms / 1e3) / 1e9
            cases.append({"N": N, "K": K, "T": T, "us": round(ms * 1e3, 2), "GB/s": round(gbs, 1),
                          "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes": int(gemv_bytes(T, N, K, RANK_R)),
                          "launches_per_call": launches,
                          "chain": chain_entry(ms_chain, gemv_bytes(T, N, K, RANK_R), peaks)})
        del ring
    status = q.get_status()
    gm = math.exp(sum(math.log(c["GB/s"]) for c in cases) / len(cases))
    print(json.dumps({"metric": "QLoRA decode-shaped linear forward, HBM GB/s (geomean over cases)",
                      "value": round(gm, 1), "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
                      "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
                      "config": {"workload": DECODE_WORKLOAD, "r": RANK_R, "alpha": ALPHA,
                                 "l2": L2_NOTE},
                      "roofline": {"bound": "hbm", "unit": "GB/s", "peak": peaks["hbm_gbs"],
                                   "peak_source": f"{kind} (HBM copy)", "achieved": round(gm, 1),
                                   "frac": round(gm / peaks["hbm_gbs"], 4)},
                      "cases": cases, "device_status": status}), flush=True)
    return 0


def run_codec_sweep(args):
    import torch
    import bit_nf4_quantized_14_b200 as q
    peaks, kind = load_peaks()
    device = torch.device("cuda", 0)
    flush = L2Flush(device)
    # the sweep tensor is drawn on the device (seeded torch generator; rows of 4096, sigma_row ~ U(0.005,
    # 0.05), 0.1 % x10 outliers), in independent 2^28-element pieces: 2^31 elements in seconds, not minutes
    chunk = 1 << 28
    nmax = max(SWEEP_SIZES)
    gen = torch.Generator(device=device)
    gen.manual_seed(50)
    x = torch.empty(nmax, dtype=torch.float32, device=device)
    for c in range(0, nmax, chunk):
        m = min(chunk, nmax - c)
        x[c:c + m] = device_sweep(m, gen)
    xb = x.to(torch.bfloat16)
    cases = []
    for n in SWEEP_SIZES:
        out = q.NF4Weight.empty(1, n, device)
        ws = torch.empty(q.quantize_workspace_bytes(n), dtype=torch.uint8, device=device)
        deq = torch.empty(1, n, dtype=torch.bfloat16, device=device)
        row = {"n": n}
        for name, src, bpe in (("quantize_fp32", x[:n].view(1, n), 4 + DEQ_B_PER_ELEM - 2),
                               ("quantize_bf16", xb[:n].view(1, n), 2 + DEQ_B_PER_ELEM - 2)):
            ms = time_calls(lambda: q.quantize(src, out=out, workspace=ws), flush, args.steps, args.warmup)
            row[name] = {"us": round(ms * 1e3, 2), "GB/s": round(n * bpe / (ms / 1e3) / 1e9, 1),
                         "frac": round(n * bpe / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4)}
        ms = time_calls(lambda: q.dequantize(out, torch.bfloat16, out=deq), flush, args.steps, args.warmup)
        row["dequantize_bf16"] = {"us": round(ms * 1e3, 2), "GB/s": round(n * DEQ_B_PER_ELEM / (ms / 1e3) / 1e9, 1),
                                  "frac": round(n * DEQ_B_PER_ELEM / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4)}
        # the variant without double quantization: fp32 constants, 0.5 + 4/64 B per element stored
        single = q.NF4SingleWeight.empty(1, n, device)
        sb = 0.5 + 4 / 64
        for name, fn, bpe in (("quantize_single_fp32", lambda: q.quantize_single(x[:n].view(1, n), out=single), 4 + sb),
                              ("dequantize_single_bf16", lambda: q.dequantize_single(single, torch.bfloat16, out=deq),
                               sb + 2)):
            ms = time_calls(fn, flush, args.steps, args.warmup)
            row[name] = {"us": round(ms * 1e3, 2), "GB/s": round(n * bpe / (ms / 1e3) / 1e9, 1),
                         "frac": round(n * bpe / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4)}
        cases.append(row)
        del out, ws, deq, single
    status = q.get_status()
    top = cases[-1]
    print(json.dumps({"metric": "NF4 quantize / dequantize HBM GB/s over the size sweep (value: fp32 quantize "
                                "at the largest size)",
                      "value": top["quantize_fp32"]["GB/s"], "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
                      "warmup": args.warmup, "higher_is_better": True, "dtype": "f32/bf16 in, u8 + e4m3 out",
                      "data": "synthetic",
                      "config": {"workload": "sweep tensors: rows of 4096, sigma_row ~ U(0.005, 0.05), 0.1 % x10 "
                                             "outliers, drawn on the device; sizes 2^20..2^31 (2^30 and 2^31 = independent 2^28 "
                                             "pieces)",
                                 "l2": L2_NOTE},
                      "roofline": {"bound": "hbm", "unit": "GB/s", "peak": peaks["hbm_gbs"],
                                   "peak_source": f"{kind} (HBM copy)"},
                      "cases": cases, "device_status": status}), flush=True)
    return 0


STUDY_SHAPE = (8192, 8192)
STUDY_LLOYD_STEPS = 30


def run_codebook_study(args):
    """The page's codebook comparison at scale through the library's kernels: an 8192 x 8192 Gaussian
    matrix (2^26 elements, 256 MB fp32, larger than L2) in blocks of 64 with fp32 constants, under
    symmetric int4, the {-8..7}/8 grid, NF4 and Lloyd's codebook (30 device steps from NF4)."""
    import numpy as np
    import torch
    import synth
    import bit_nf4_quantized_14_b200 as q
    peaks, kind = load_peaks()
    device = torch.device("cuda", 0)
    flush = L2Flush(device)
    x = torch.from_numpy(synth.normal_f32(STUDY_SHAPE, 1.0, 0, 17).reshape(-1)).to(device)
    n = x.numel()
    nf4, _ = q.codebook()
    codes = torch.empty(-(-n // 2), dtype=torch.uint8, device=device)
    absmax = torch.empty(-(-n // 64), dtype=torch.float32, device=device)
    out32 = torch.empty(n, dtype=torch.float32, device=device)
    st = torch.empty(q.CODEBOOK_STATS_LEN, dtype=torch.float64, device=device)
    ws = torch.empty(q.codebook_stats_workspace_bytes(n), dtype=torch.uint8, device=device)
    stored = 0.5 + 4 / 64
    for _ in range(args.warmup):
        q.lloyd(x, nf4, 1)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record()
    lloyd_lv, hist = q.lloyd(x, nf4, STUDY_LLOYD_STEPS)
    t1.record()
    torch.cuda.synchronize()
    lloyd_ms = t0.elapsed_time(t1) / (STUDY_LLOYD_STEPS + 1)
    books = {"int4_symmetric": np.arange(-7, 8, dtype=np.float32) / np.float32(7),
             "grid_16": np.arange(-8, 8, dtype=np.float32) / np.float32(8), "nf4": nf4, "lloyd": lloyd_lv}
    cases = {}
    for name, lv in books.items():
        row = {"levels": [float(v) for v in lv]}
        for label, fn, bpe in (
                ("quantize", lambda: q.codebook_quantize(x, lv, codes, absmax), 4 + stored),
                ("dequantize_fp32", lambda: q.codebook_dequantize(codes, absmax, n, lv, torch.float32, out32), stored + 4),
                ("stats", lambda: q.codebook_stats(x, codes, absmax, lv, st, ws), 4 + stored)):
            ms = time_calls(fn, flush, args.steps, args.warmup)
            row[label] = {"us": round(ms * 1e3, 2), "GB/s": round(n * bpe / (ms / 1e3) / 1e9, 1),
                          "frac": round(n * bpe / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4)}
        q.codebook_quantize(x, lv, codes, absmax)
        d = q.stats_dict(q.codebook_stats(x, codes, absmax, lv, st, ws), lv.size)
        row.update(entropy_bits=round(d["entropy_bits"], 4), rms=d["rms"])
        cases[name] = row
    figures = {
        "entropy_bits_nf4": cases["nf4"]["entropy_bits"],
        "entropy_bits_int4_symmetric": cases["int4_symmetric"]["entropy_bits"],
        "rms_reduction_nf4_vs_int4": round(1 - cases["nf4"]["rms"] / cases["int4_symmetric"]["rms"], 4),
        "lloyd_gain_over_nf4": round(1 - cases["lloyd"]["rms"] / cases["nf4"]["rms"], 4),
        "page": {"entropy_bits_nf4": 3.88, "entropy_bits_int4_symmetric": 3.50, "rms_reduction_nf4_vs_int4": 0.15,
                 "lloyd_gain_over_nf4": 0.05}}
    status = q.get_status()
    print(json.dumps({"metric": "Lloyd step (codebook quantize + statistics) throughput on the codebook "
                                "comparison matrix",
                      "value": round(n / (lloyd_ms / 1e3) / 1e9, 2), "unit": "G elements/s", "n_gpus": 1,
                      "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
                      "ms_per_lloyd_step": round(lloyd_ms, 4), "dtype": "f32 in, u8 codes + fp32 constants, f64 sums",
                      "data": "synthetic",
                      "config": {"workload": "8192 x 8192 N(0, 1) fp32 matrix (2^26 elements), blocks of 64, fp32 "
                                             "constants; codebooks int4 {-7..7}/7, grid {-8..7}/8, NF4, Lloyd "
                                             f"({STUDY_LLOYD_STEPS} device steps from NF4)",
                                 "l2": L2_NOTE + " (codec calls); the Lloyd loop runs "
                                       "back to back (input 256 MB > L2)"},
                      "roofline": {"bound": "hbm", "unit": "GB/s", "peak": peaks["hbm_gbs"],
                                   "peak_source": f"{kind} (HBM copy)"},
                      "figures": figures, "rms_history": hist, "cases": cases, "device_status": status}), flush=True)
    return 0


LLAMA65B_LAYERS, LLAMA65B_TOKENS = 80, 512
LLAMA65B_WORKLOAD = ("LLaMA-65B-shaped decoder linears: 80 layers x (q, k, v, o 8192x8192; gate, up 22016x8192; "
                     "down 8192x22016) as NF4 + LoRA r = 64, alpha = 16; one step = the 560 linear forward + "
                     "backward calls at T = 1 x 512 tokens (the hot-path part of a QLoRA training step)")


def run_llama65b(args):
    """All 80 layers' NF4 weights resident (33.4 GB); weights, adapters and activations are seeded
    device-side normal draws (random init, no checkpoint)."""
    import torch
    import bit_nf4_quantized_14_b200 as q
    peaks, kind = load_peaks()
    device = torch.device("cuda", 0)
    gen = torch.Generator(device=device)
    gen.manual_seed(65)
    per_layer = [(8192, 8192)] * 4 + [(22016, 8192)] * 2 + [(8192, 22016)]
    T = LLAMA65B_TOKENS
    layers = []
    for _ in range(LLAMA65B_LAYERS):
        lin = []
        for N, K in per_layer:
            W = torch.randn(N, K, device=device, generator=gen).mul_(0.02)
            nf4 = q.quantize(W)
            del W
            A = (torch.randn(RANK_R, K, device=device, generator=gen) * 0.01).to(torch.bfloat16)
            B = (torch.randn(N, RANK_R, device=device, generator=gen) * 0.01).to(torch.bfloat16)
            lin.append((N, K, nf4, A, B))
        layers.append(lin)
    bufs = {}
    for N, K in set(per_layer):
        bufs[(N, K)] = dict(
            X=torch.randn(T, K, device=device, generator=gen).to(torch.bfloat16),
            dY=torch.randn(T, N, device=device, generator=gen).to(torch.bfloat16),
            Y=torch.empty(T, N, dtype=torch.bfloat16, device=device),
            U=torch.empty(T, RANK_R, dtype=torch.bfloat16, device=device),
            dX=torch.empty(T, K, dtype=torch.bfloat16, device=device),
            dA=torch.empty(RANK_R, K, dtype=torch.float32, device=device),
            dB=torch.empty(N, RANK_R, dtype=torch.float32, device=device),
            ws=torch.empty(q.linear_workspace_bytes(T, N, K, RANK_R), dtype=torch.uint8, device=device))

    def step():
        for lin in layers:
            for N, K, nf4, A, B in lin:
                b = bufs[(N, K)]
                q.linear_fwd(b["X"], nf4, A, B, ALPHA, out=b["Y"], U_out=b["U"], workspace=b["ws"])
                q.linear_bwd(b["dY"], b["X"], nf4, A, B, ALPHA, U=b["U"], dX=b["dX"], dA=b["dA"], dB=b["dB"],
                             workspace=b["ws"])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    q.profile_read()
    q.profile_enable(True)
    clocks = ClockSampler(0)
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = q.kernel_launches()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    while not ev1.query():
        time.sleep(0.0005)
    torch.cuda.synchronize()
    launches = q.kernel_launches() - n0
    clk = clocks.stop()
    q.profile_enable(False)
    prof = q.profile_read()
    ms = ev0.elapsed_time(ev1)
    flops = LLAMA65B_LAYERS * sum(fwd_flops(T, N, K, RANK_R) + bwd_flops(T, N, K, RANK_R) for N, K in per_layer)
    value = flops * args.steps / (ms / 1e3) / 1e12
    peak = peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]
    parts = {c: {"launches": n, "ms_total": round(t, 3)} for c, (n, t) in prof.items()}
    print(json.dumps({"metric": "QLoRA linear fwd+bwd TFLOP/s, LLaMA-65B-shaped step (560 linears at T = 512)",
                      "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
                      "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True,
                      "dtype": "bf16", "data": "synthetic (device-side seeded normals, random init)",
                      "config": {"workload": LLAMA65B_WORKLOAD, "tokens": T, "r": RANK_R, "alpha": ALPHA,
                                 "l2": "no flush: one step streams 33.4 GB of NF4 weights"},
                      "roofline": {"bound": "tensor", "unit": "TFLOP/s", "peak": peak,
                                   "peak_source": f"{kind} (sustained bf16)", "achieved": round(value, 3),
                                   "frac": round(value / peak, 4)},
                      "gpu_launches": int(launches), "parts": parts, "clocks": clk,
                      "device_status": q.get_status()}), flush=True)
    return 0


LLAMA65B_TRAIN_WORKLOAD = ("LLaMA-65B-shaped QLoRA training step: token embedding, 80 decoder layers (RMSNorm, causal "
                           "attention with 64 heads over NF4+LoRA q/k/v/o, RMSNorm, SwiGLU over NF4+LoRA gate/up/"
                           "down), final RMSNorm, bf16 output head, cross-entropy on uniform random targets, AdamW "
                           "on the fp32 LoRA adapters (r = 64, alpha = 16); batch 1 x 512 tokens, vocab 32000, "
                           "random init")


def lora_param_count(layers=80, d=8192, ffn=22016, r=64):
    per_layer = 4 * (r * d + d * r) + 2 * (r * d + ffn * r) + (r * ffn + d * r)
    return layers * per_layer


def run_paged_adamw(args):
    """The paged optimizer's step over the LoRA adapters of the LLaMA-65B-shaped model (r = 64 on all
    seven linears of 80 layers: 0.80 G fp32 parameters, 6.4 GB of AdamW moments), with the moments in
    device memory, in managed memory resident on the GPU, and in managed memory evicted to the host
    before the step (paged back by the kernel's own accesses, or by an explicit prefetch first)."""
    import torch
    import bit_nf4_quantized_14_b200 as q
    peaks, kind = load_peaks()
    device = torch.device("cuda", 0)
    gen = torch.Generator(device=device)
    gen.manual_seed(77)
    n = lora_param_count()
    p = torch.randn(n, device=device, generator=gen).mul_(0.02)
    g = torch.randn(n, device=device, generator=gen).mul_(1e-3)
    stream = torch.cuda.current_stream()

    def timed(fn, before=None, steps=args.steps):
        ts = []
        for k in range(args.warmup + steps):
            if before is not None:
                before()
                torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn(k + 1)
            e1.record(stream)
            e1.synchronize()
            if k >= args.warmup:
                ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    md = torch.zeros(n, device=device)
    vd = torch.zeros(n, device=device)
    n0 = q.kernel_launches()
    ms_dev = timed(lambda t: q.adamw_step(p, g, md, vd, t, 2e-4))
    launches_dev = (q.kernel_launches() - n0) / (args.warmup + args.steps)
    del md, vd
    mp, vp = q.paged_empty(n, device), q.paged_empty(n, device)
    mp.zero_()
    vp.zero_()
    q.paged_prefetch(mp, True)
    q.paged_prefetch(vp, True)
    torch.cuda.synchronize()
    ms_res = timed(lambda t: q.adamw_step(p, g, mp, vp, t, 2e-4))

    def evict():
        q.paged_prefetch(mp, False)
        q.paged_prefetch(vp, False)

    few = max(1, min(args.steps, 5))
    ms_fault = timed(lambda t: q.adamw_step(p, g, mp, vp, t, 2e-4), before=evict, steps=few)

    def prefetch_then_step(t):
        q.paged_prefetch(mp, True)
        q.paged_prefetch(vp, True)
        q.adamw_step(p, g, mp, vp, t, 2e-4)

    ms_pref = timed(prefetch_then_step, before=evict, steps=few)
    del mp, vp
    tp = torch.nn.Parameter(p.clone())
    tp.grad = g.clone()
    topt = torch.optim.AdamW([tp], lr=2e-4, weight_decay=0.0, fused=True)
    ms_torch = timed(lambda t: topt.step())
    status = q.get_status()
    bpp = 28
    gbs = n * bpp / (ms_res / 1e3) / 1e9
    mig = 8 * n
    print(json.dumps({"metric": "paged AdamW step over the LLaMA-65B-shaped LoRA adapters (moments in managed memory)",
                      "value": round(ms_res, 3), "unit": "ms per optimizer step", "n_gpus": 1, "steps": args.steps,
                      "warmup": args.warmup, "higher_is_better": False, "dtype": "f32",
                      "data": "synthetic (random parameters and gradients)",
                      "config": {"workload": "AdamW over 0.80 G fp32 LoRA parameters (r = 64, all seven linears of "
                                             "80 LLaMA-65B layers), lr 2e-4, betas (0.9, 0.999), eps 1e-8",
                                 "params": n, "state_bytes": mig,
                                 "l2": "inputs (22 GB per step) far above L2"},
                      "roofline": {"bound": "hbm", "unit": "GB/s", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                                   "frac": round(gbs / peaks["hbm_gbs"], 4), "kernel": "adamw_kernel (resident states)",
                                   "algorithmic_bytes_per_param": bpp, "peak_source": f"{kind} (HBM copy)"},
                      "cases_ms": {"device_states": round(ms_dev, 3), "managed_resident": round(ms_res, 3),
                                   "managed_evicted_demand_paged": round(ms_fault, 3),
                                   "managed_evicted_prefetch_then_step": round(ms_pref, 3),
                                   "torch_fused_adamw_device_states": round(ms_torch, 3)},
                      "page_in_GBps": {"demand_paged": round(mig / ((ms_fault - ms_res) / 1e3) / 1e9, 1),
                                       "prefetch": round(mig / ((ms_pref - ms_res) / 1e3) / 1e9, 1)},
                      "gpu_launches": launches_dev, "device_status": status}), flush=True)
    return 0


def build_decoder(layers, d, ffn, heads, vocab, r, gen, device):
    """A LLaMA-shaped decoder whose seven linears per layer are QLoRALinear modules (random init)."""
    import torch
    from bit_nf4_quantized_14_b200.autograd import QLoRALinear

    def lin(n, k):
        w = torch.randn(n, k, device=device, generator=gen).mul_(0.02)
        m = QLoRALinear(w, r=r, alpha=ALPHA, generator=gen)
        del w
        return m

    class Layer(torch.nn.Module):
        def __init__(self):
            super().__init__()
            self.q, self.k, self.v, self.o = lin(d, d), lin(d, d), lin(d, d), lin(d, d)
            self.gate, self.up, self.down = lin(ffn, d), lin(ffn, d), lin(d, ffn)
            self.n1 = torch.ones(d, device=device, dtype=torch.bfloat16)
            self.n2 = torch.ones(d, device=device, dtype=torch.bfloat16)

        def forward(self, h):
            T = h.shape[0]
            x = rms(h, self.n1)
            q = self.q(x).view(T, heads, d // heads).transpose(0, 1)
            k = self.k(x).view(T, heads, d // heads).transpose(0, 1)
            v = self.v(x).view(T, heads, d // heads).transpose(0, 1)
            a = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], is_causal=True)[0]
            h = h + self.o(a.transpose(0, 1).reshape(T, d))
            x = rms(h, self.n2)
            return h + self.down(torch.nn.functional.silu(self.gate(x)) * self.up(x))

    def rms(x, w, eps=1e-5):
        xf = x.float()
        return (xf * torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + eps)).to(torch.bfloat16) * w

    class Decoder(torch.nn.Module):
        def __init__(self):
            super().__init__()
            self.emb = (torch.randn(vocab, d, device=device, generator=gen) * 0.02).to(torch.bfloat16)
            self.layers = torch.nn.ModuleList([Layer() for _ in range(layers)])
            self.nf = torch.ones(d, device=device, dtype=torch.bfloat16)
            self.head = (torch.randn(vocab, d, device=device, generator=gen) * 0.02).to(torch.bfloat16)

        def forward(self, ids, targets):
            h = self.emb[ids]
            for layer in self.layers:
                h = layer(h)
            logits = rms(h, self.nf) @ self.head.t()
            return torch.nn.functional.cross_entropy(logits.float(), targets)

    return Decoder()


def run_llama65b_train(args):
    import torch
    import bit_nf4_quantized_14_b200 as q
    device = torch.device("cuda", 0)
    gen = torch.Generator(device=device)
    gen.manual_seed(66)
    vocab, T = 32000, LLAMA65B_TOKENS
    model = build_decoder(LLAMA65B_LAYERS, 8192, 22016, 64, vocab, RANK_R, gen, device)
    params = [p for p in model.parameters() if p.requires_grad]
    if args.optimizer == "torch":
        opt = torch.optim.AdamW(params, lr=2e-4, weight_decay=0.0, fused=True)
    else:
        from bit_nf4_quantized_14_b200.optim import PagedAdamW
        opt = PagedAdamW(params, lr=2e-4, weight_decay=0.0, paged=True)
    ids = torch.randint(0, vocab, (T,), device=device, generator=gen)
    targets = torch.randint(0, vocab, (T,), device=device, generator=gen)

    def step():
        if args.optimizer == "paged_evicted":
            opt.evict_states()          # a memory spike pushed the moments out; the step pages them back
        elif args.optimizer == "paged_evicted_prefetch":
            opt.prefetch_states_async(evict_first=True)   # the same spike, then the moments are brought
                                                          # back while the forward and backward run
        loss = model(ids, targets)
        loss.backward()
        opt.step()
        if args.optimizer == "torch":
            opt.zero_grad(set_to_none=True)
        else:
            opt.zero_grad()
        return loss

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    q.profile_read()
    q.profile_enable(True)
    clocks = ClockSampler(0)
    clocks.start()
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = q.kernel_launches()
    ev0.record(stream)
    for _ in range(args.steps):
        loss = step()
    ev1.record(stream)
    while not ev1.query():
        time.sleep(0.0005)
    torch.cuda.synchronize()
    launches = q.kernel_launches() - n0
    clk = clocks.stop()
    q.profile_enable(False)
    prof = q.profile_read()
    ms = ev0.elapsed_time(ev1) / args.steps
    lin_ms = sum(prof[c][1] for c in ("fwd_gemm", "bwd_gemm", "lora")) / args.steps
    n_lora = sum(p.numel() for p in params)
    print(json.dumps({"metric": "QLoRA training step, LLaMA-65B-shaped, tokens/s",
                      "value": round(T / (ms / 1e3), 1), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
                      "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
                      "dtype": "bf16 (NF4 weights, fp32 adapters)", "data": "synthetic (random init, random ids)",
                      "config": {"workload": LLAMA65B_TRAIN_WORKLOAD, "tokens": T, "r": RANK_R, "alpha": ALPHA,
                                 "lora_params": n_lora, "nf4_weight_bytes": sum(
                                     m.w.nbytes for m in model.modules() if hasattr(m, "w"))},
                      "optimizer": {"torch": "torch.optim.AdamW (fused, device states)",
                                    "paged": "PagedAdamW (library kernel, moments in managed memory, resident)",
                                    "paged_evicted": "PagedAdamW, moments evicted to the host at the start of every "
                                                     "step and paged back by the optimizer step",
                                    "paged_evicted_prefetch": "PagedAdamW, moments evicted at the start of every "
                                                              "step on a side stream and prefetched back there "
                                                              "while the forward and backward run"}[args.optimizer],
                      "library_linears_ms_per_step": round(lin_ms, 3),
                      "library_linears_share": round(lin_ms / ms, 4),
                      "final_loss": float(loss.item()), "gpu_launches": int(launches), "clocks": clk,
                      "device_status": q.get_status()}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffer) measurement")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the decode and codec figures carried in the headline line")
    ap.add_argument("--optimizer", choices=["torch", "paged", "paged_evicted", "paged_evicted_prefetch"],
                    default="torch",
                    help="with --workload llama65b_train: the adapters' optimizer")
    ap.add_argument("--workload", choices=["llama7b_step", "decode", "codec_sweep", "llama65b_linears",
                                           "llama65b_train", "codebook_study", "paged_adamw", "flush_check"],
                    default="llama7b_step",
                    help="llama7b_step (the headline line), or the decode / codec-sweep / 65B-step measurement lines")
    ap.add_argument("--ncu-summary", metavar="CSV", default=None,
                    help="summarise an ncu launch list (time + DRAM bytes per launch) and write profiles/traffic.json")
    ap.add_argument("--ncu-last", type=int, default=96, help="with --ncu-summary: launches to summarise (the last N)")
    ap.add_argument("--ncu-calls", type=int, default=6, help="with --ncu-summary: timed calls of each class in them")
    ap.add_argument("--ncu-command", default="", help="with --ncu-summary: the command the list came from")
    ap.add_argument("--shapes", default="all",
                    help="comma-separated NxK subset of the workload shapes (profiling runs), e.g. 4096x4096")
    args = ap.parse_args(argv)
    if args.shapes != "all":
        global SHAPES
        SHAPES = [tuple(int(v) for v in sh.split("x")) for sh in args.shapes.split(",")]
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.ncu_summary:
        return ncu_summary(args.ncu_summary, args.ncu_last, args.ncu_calls, args.ncu_command)
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "decode":
        return run_decode(args)
    if args.workload == "codec_sweep":
        return run_codec_sweep(args)
    if args.workload == "llama65b_linears":
        return run_llama65b(args)
    if args.workload == "llama65b_train":
        return run_llama65b_train(args)
    if args.workload == "codebook_study":
        return run_codebook_study(args)
    if args.workload == "paged_adamw":
        return run_paged_adamw(args)
    if args.workload == "flush_check":
        return run_flush_check(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
