"""Benchmark of the microscaling-FP4 hot path on B200.

Default workload (the one the headline metric is quoted on): NVFP4 quantize and
dequantize of a 4096 x 4096 bf16 tensor drawn from 0.1 * Student-t(3) (seed 1),
16-element E4M3 blocks under an fp32 tensor scale, run twice -- round-to-nearest
and Philox stochastic rounding (seed 1) -- each followed by an fp32 dequantize.
One step = tensor amax + RTN quantize + dequantize + SR quantize + dequantize.

Other workloads (--workload, for measurement only): mx_linear_128x512,
hadamard_mxfp4_gemm (rotate+quantize X[8192,4096] then GEMM against
W[11008,4096] -> bf16), vit_b16_linears (fwd/dgrad/wgrad of qkv/fc1/fc2 at
M = 50432), llama7b_nvfp4 (amax + quantize + GEMM over the Llama-7B shapes).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fp4|reference] [--workload NAME]

Prints one JSON line on rank 0.  Device time is taken with CUDA events on the
launching stream, bracketed by a barrier and synchronize, max over ranks.  With
N > 1 every rank runs its own copy of the workload (weak scaling, no data-path
collective).  `--impl reference` times the CPU oracle on this machine's host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantize+rotate HBM GB/s; block-scaled FP4 GEMM TFLOP/s; % of roofline"


# ----------------------------------------------------------------- helpers ---

def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples (every 100 ms) with host timestamps, kept for the timed window."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.samples = []
        self.proc = None
        self.gpu = gpu_index
        self.t_start = self.t_end = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [s.strip() for s in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        inside = [s for t, s in self.samples if self.t_start <= t <= self.t_end]
        used = inside if inside else [min(self.samples, key=lambda ts: abs(ts[0] - self.t_end))[1]]
        sm = [float(s[0]) for s in used if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in used if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for s in used for n, v in zip(names, s[4:8]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(inside)}


class KernelTimer:
    """CUDA-event timing of one kernel family inside the timed region."""

    def __init__(self, torch):
        self.torch = torch
        self.pairs = []

    def around(self, fn):
        t = self.torch
        a = t.cuda.Event(enable_timing=True)
        b = t.cuda.Event(enable_timing=True)
        a.record()
        out = fn()
        b.record()
        self.pairs.append((a, b))
        return out

    def mean_ms(self):
        if not self.pairs:
            return None
        return float(np.mean([a.elapsed_time(b) for a, b in self.pairs]))


# -------------------------------------------------------------- workloads ---

class NvfpStudentT:
    """NVFP4 quantize (RTN, then Philox SR) + fp32 dequantize of 0.1*Student-t(3), 4096x4096."""

    name = "nvfp4_student_t_4096"
    rows = cols = 4096
    n_inputs = 4                 # rotating input copies: 128 MB of inputs, each step writes ~146 MB
    launches_per_step = 5        # amax, quantize RTN, dequantize, quantize SR, dequantize
    unit = "GB/s"

    def __init__(self, torch, F):
        self.t, self.F = torch, F
        n = self.rows * self.cols
        self.n = n
        # algorithmic HBM bytes per element: quantize = 2 (bf16 in) + 0.5 (codes) + 1/16 (E4M3 scales);
        # dequantize = 0.5 + 1/16 in + 4 (fp32) out.  The tensor amax needs x once more, which the
        # method can serve from L2 (32 MB < 126 MB), so it adds no algorithmic bytes.
        self.q_bytes = n * (2 + 0.5 + 1 / 16)
        self.d_bytes = n * (0.5 + 1 / 16 + 4)
        self.step_bytes = 2 * self.q_bytes + 2 * self.d_bytes

    def setup(self, device):
        from workloads import nvfp4_student_t
        t = self.t
        bits = nvfp4_student_t(self.rows, self.cols, seed=1)
        self.host_bits = bits
        base = t.from_numpy(bits.view(np.int16)).view(t.bfloat16)
        self.x = [base.to(device).clone() for _ in range(self.n_inputs)]
        self.codes = [t.empty((self.rows, self.cols // 2), dtype=t.uint8, device=device) for _ in range(2)]
        self.scales = [t.empty((self.rows, self.cols // 16), dtype=t.uint8, device=device) for _ in range(2)]
        self.ts = t.empty((1,), dtype=t.float32, device=device)
        self.ts_sr = t.empty((1,), dtype=t.float32, device=device)
        self.deq = [t.empty((self.rows, self.cols), dtype=t.float32, device=device) for _ in range(2)]
        # "amax+quantize_rtn" covers two kernels (the entry point launches the amax pass first);
        # the others time exactly one kernel each and are the roofline candidates.
        self.timers = {k: KernelTimer(t) for k in ("amax+quantize_rtn", "quantize_sr", "dequantize")}
        self.single_kernel = ("quantize_sr", "dequantize")

    def step(self, i, timed=False, x=None):
        F = self.F
        x = self.x[i % self.n_inputs] if x is None else x
        T = self.timers if timed else None

        def run(key, fn):
            return T[key].around(fn) if T is not None else fn()

        # RTN: tensor amax + quantize (one entry point), then dequantize
        run("amax+quantize_rtn", lambda: F.fp4_quantize(x, fmt="nvfp4", rnd="rtn", codes=self.codes[0],
                                                   scales=self.scales[0], tensor_scale_out=self.ts))
        run("dequantize", lambda: F.fp4_dequantize(self.codes[0], self.scales[0], self.ts, fmt="nvfp4",
                                                   out=self.deq[0]))
        # SR with the same tensor scale, then dequantize
        run("quantize_sr", lambda: F.fp4_quantize(x, fmt="nvfp4", rnd="sr", seed=1, tensor_scale_in=self.ts,
                                                  codes=self.codes[1], scales=self.scales[1],
                                                  tensor_scale_out=self.ts_sr))
        run("dequantize", lambda: F.fp4_dequantize(self.codes[1], self.scales[1], self.ts_sr, fmt="nvfp4",
                                                   out=self.deq[1]))

    def outputs(self):
        return [self.codes[0], self.scales[0], self.ts, self.deq[0], self.codes[1], self.scales[1], self.ts_sr,
                self.deq[1]]

    def kernel_bytes(self, key):
        return self.q_bytes if key.startswith("quantize") else self.d_bytes

    def value_from_ms(self, ms_per_step, n_ranks):
        return self.step_bytes * n_ranks / (ms_per_step * 1e-3) / 1e9

    def config(self):
        return {"workload": self.name, "shape": [self.rows, self.cols], "format": "nvfp4", "block": 16,
                "distribution": "0.1*student_t(3)", "seed": 1, "rounding": ["rtn", "sr(philox4x32-10, seed 1)"],
                "dequantize": "f32", "algorithmic_bytes_per_step": self.step_bytes,
                "l2": f"{self.n_inputs} rotating input copies (128 MB) and ~146 MB written per step"}

    # ---- CPU oracle on the same workload ----
    def oracle_step(self, rows):
        import oracle as O
        from workloads import bf16_to_f32
        x32 = bf16_to_f32(self.host_bits[:rows]) if rows < self.rows else bf16_to_f32(self.host_bits)
        s_t = O.nv_tensor_scale(bf16_to_f32(self.host_bits))
        r = O.quantize_values(x32, fmt="nvfp4", rnd="rtn", tensor_scale=s_t)
        O.dequantize(r["codes"], r["scales"], fmt="nvfp4", tensor_scale=s_t)
        r = O.quantize_values(x32, fmt="nvfp4", rnd="sr", seed=1, tensor_scale=s_t)
        O.dequantize(r["codes"], r["scales"], fmt="nvfp4", tensor_scale=s_t)
        return rows * self.cols * (2 * (2 + 0.5 + 1 / 16) + 2 * (0.5 + 1 / 16 + 4))


WORKLOADS = {NvfpStudentT.name: NvfpStudentT}


# ------------------------------------------------------------------ arms ---

def _dist_setup(torch):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local, pg


def _max_over_ranks(torch, pg, value: float) -> float:
    """Max of a per-rank scalar over the process group (device time: the slowest rank counts)."""
    if pg is None:
        return value
    dev = "cuda" if pg.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def _barrier(torch, pg):
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()


def run_fp4(args):
    import torch
    import microscaling_fp4_quantization_mxfp4_b200 as F
    from microscaling_fp4_quantization_mxfp4_b200 import _lib
    _lib.load()                                  # fail loudly when the CUDA library is missing
    ws, rank, local, pg = _dist_setup(torch)
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    W = WORKLOADS[args.workload](torch, F)
    W.setup(device)

    for i in range(args.warmup):
        W.step(i)
    F.fp4_check_device_errors()

    sampler = ClockSampler(_smi_id(torch, local))
    sampler.start()
    time.sleep(0.3)                              # let the sampler produce its first line
    _barrier(torch, pg)
    sampler.t_start = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(args.steps):
        W.step(i, timed=True)
    end.record()
    torch.cuda.synchronize()
    sampler.t_end = time.time()
    _barrier(torch, pg)
    sampler.stop()
    F.fp4_check_device_errors()
    ms_total = _max_over_ranks(torch, pg, start.elapsed_time(end))
    ms_step = ms_total / args.steps
    value = W.value_from_ms(ms_step, ws)

    # dominant kernel: largest share of device time in the timed region
    per = {k: (tm.mean_ms(), len(tm.pairs)) for k, tm in W.timers.items() if tm.pairs}
    dom = max((k for k in per if k in W.single_kernel), key=lambda k: per[k][0] * per[k][1])
    dom_ms = _max_over_ranks(torch, pg, per[dom][0])
    peaks = _peaks()
    achieved = W.kernel_bytes(dom) / (dom_ms * 1e-3) / 1e9
    traffic = _load_traffic(W.name, dom)
    roofline = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic, "peak_source": peaks["source"],
                "per_kernel_us": {k: round(v[0] * 1e3, 2) for k, v in per.items()}}

    # end to end through the public API with host buffers: pinned H2D of the input, the step,
    # D2H of every output (codes, scales, tensor scales, dequantized tensors)
    host_in = torch.from_numpy(W.host_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    dev_in = torch.empty_like(W.x[0])
    outs = W.outputs()
    host_outs = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
    h2d = host_in.numel() * host_in.element_size()
    d2h = sum(o.numel() * o.element_size() for o in outs)
    e2e_steps = max(3, min(20, args.steps))
    for _ in range(2):
        dev_in.copy_(host_in, non_blocking=True)
        W.step(0, x=dev_in)
        for h, o in zip(host_outs, outs):
            h.copy_(o, non_blocking=True)
    _barrier(torch, pg)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        dev_in.copy_(host_in, non_blocking=True)
        W.step(0, x=dev_in)
        for h, o in zip(host_outs, outs):
            h.copy_(o, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(torch, pg, e0.elapsed_time(e1)) / e2e_steps
    e2e = {"value": round(W.value_from_ms(e2e_ms, ws), 2), "unit": W.unit, "ms_per_step": round(e2e_ms, 4),
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = _cpu_baseline(W)
    clocks = sampler.summary()
    if pg is not None:
        pg.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": W.unit, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded NumPy PCG64, bf16)",
        "config": dict(W.config(), parallelism=f"replicas{ws}" if ws > 1 else "single"),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": W.launches_per_step * args.steps, "clocks": clocks, "impl": "fp4",
    }
    print(json.dumps(line), flush=True)


def _smi_id(torch, local):
    """nvidia-smi -i selector of this process's GPU (its UUID; the index as a fallback)."""
    try:
        u = str(torch.cuda.get_device_properties(local).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(local)


KERNEL_SOURCES = ["microscaling_fp4_quantization_mxfp4_b200/csrc/quantize.cu",
                  "microscaling_fp4_quantization_mxfp4_b200/csrc/fp4_device.cuh"]


def _sources_hash(files=KERNEL_SOURCES):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _load_traffic(workload, kernel):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu capture
    (profiles/traffic.json), or None when none exists or the kernel sources changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(workload, {}).get(kernel)
    if not d or d.get("sources_sha256_16") != _sources_hash():
        return None
    return d["dram_bytes_per_launch"]


def _cpu_baseline(W):
    """The oracle as it stands, on the whole workload (one step), on the host cores."""
    t0 = time.time()
    nbytes = W.oracle_step(W.rows)
    dt = time.time() - t0
    return {"value": round(nbytes / dt / 1e9, 4), "unit": W.unit, "cores": 1, "kind": "oracle",
            "sample": f"one full step ({W.rows}x{W.cols}) on the host, NumPy elementwise (1 thread)",
            "seconds": round(dt, 2), "host_cpus": os.cpu_count()}


def run_reference(args):
    """The oracle as the reference arm: bounded samples of the same workload on host cores."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch  # noqa: F401  (only for the shared workload classes)
    W = WORKLOADS[args.workload](None, None)
    from workloads import nvfp4_student_t
    W.host_bits = nvfp4_student_t(W.rows, W.cols, seed=1)
    rows = 256                                   # each step: 256 of 4096 rows, ~0.3 s of CPU work
    for _ in range(args.warmup):
        W.oracle_step(rows)
    t0 = time.time()
    nbytes = 0.0
    for _ in range(args.steps):
        nbytes += W.oracle_step(rows)
    dt = time.time() - t0
    value = nbytes / dt / 1e9
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": W.unit, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded NumPy PCG64, bf16)",
        "config": dict(W.config(), parallelism="single"), "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": W.unit, "kind": "oracle", "cores": 1,
                         "sample": f"{rows} of {W.rows} rows per step (global tensor scale), NumPy 1 thread"},
        "e2e": {"value": round(value, 4), "unit": W.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="fp4", choices=["fp4", "reference"])
    ap.add_argument("--workload", default=NvfpStudentT.name, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_fp4(args)


if __name__ == "__main__":
    main()
