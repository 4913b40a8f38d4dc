"""Benchmark of the microscaling-FP4 hot path on B200.

Default workload (the one the headline metric is quoted on): NVFP4 quantize and
dequantize of a 4096 x 4096 bf16 tensor drawn from 0.1 * Student-t(3) (seed 1),
16-element E4M3 blocks under an fp32 tensor scale, run twice -- round-to-nearest
and Philox stochastic rounding (seed 1) -- each followed by an fp32 dequantize.
One step = tensor amax + RTN quantize + dequantize + SR quantize + dequantize.

Other workloads (--workload; value in TFLOP/s of GEMM work per step):
  mx_linear_128x512                    quantize X[128,512], W[512,512] + GEMM, fp32 out
  hadamard_mxfp4_gemm_8192x11008x4096  rotate+quantize X[8192,4096] (b = 16/32/64/128) then
                                       GEMM against the offline-rotated W[11008,4096], bf16 out
  vit_b16_linears_50432                fwd/dgrad/wgrad of qkv/fc1/fc2 at M = 50432 with the six
                                       operand quantizations per layer (two along axis 0)
  llama7b_nvfp4_sweep                  amax + quantize + GEMM over the Llama-7B shapes and
                                       M = 1 .. 16384 (per-case times, L2 flushed between cases)

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

    def summary(self, t_start=None, t_end=None):
        """Median SM clock, max clock and active throttle reasons over the samples taken inside
        [t_start, t_end] (default: the main timed window); the nearest sample if none fell inside."""
        t_start = self.t_start if t_start is None else t_start
        t_end = self.t_end if t_end is None else t_end
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        inside = [s for t, s in self.samples if t_start <= t <= t_end]
        used = inside if inside else [min(self.samples, key=lambda ts: abs(ts[0] - t_end))[1]]
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

class Workload:
    """One synthetic workload: device setup, one step of the hot path, its algorithmic work."""

    unit = "GB/s"
    bracket = True               # step time = events around all steps (False: sum of per-case events)
    flush_between_cases = False

    def family_bound(self, key):
        return "hbm"

    def single_kernel(self):
        return ()

    def e2e_step(self):
        """One step from pinned host inputs to host outputs; returns (h2d bytes, d2h bytes)."""
        raise NotImplementedError


class NvfpStudentT(Workload):
    """NVFP4 quantize + fp32 dequantize of 0.1*Student-t(3), 4096x4096, once with RTN and once with
    Philox SR: each one fp4_quantize_dequantize launch (codes, scales and dequantized values)."""

    name = "nvfp4_student_t_4096"
    fmt = "nvfp4"                # the quantizer's format ("nvfp4_4o6": four-over-six block scales)
    fused_deq = True             # quantize and dequantize in one launch (fp4_quantize_dequantize)
    rows = cols = 4096
    n_inputs = 4                 # rotating input copies: 128 MB of inputs, each step writes ~146 MB
    launches_per_step = 2        # single-pass amax + quantize + dequantize (RTN), quantize + dequantize (SR)
    unit = "GB/s"
    gemm_companion = True        # the line also carries the GEMM half of the metric (b = 128 Hadamard GEMM)

    def __init__(self, torch, F):
        self.t, self.F = torch, F
        n = self.rows * self.cols
        self.n = n
        # algorithmic HBM bytes per element: quantize = 2 (bf16 in) + 0.5 (codes) + 1/16 (E4M3 scales);
        # dequantize = 4 (fp32) out, plus 0.5 + 1/16 in when it is a separate pass over the codes.
        # The tensor amax needs x once more, which the method can serve from L2 (32 MB < 126 MB),
        # so it adds no algorithmic bytes.
        self.q_bytes = n * (2 + 0.5 + 1 / 16)
        self.d_bytes = n * (4 if self.fused_deq else 0.5 + 1 / 16 + 4)
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
        # "amax+quantize_rtn" covers the single-pass amax+quantize kernel (two kernels when the
        # tensor does not fit the single pass); the others time exactly one kernel per launch.
        keys = ("amax+quantize_dequantize_rtn", "quantize_dequantize_sr") if self.fused_deq else \
            ("amax+quantize_rtn", "quantize_sr", "dequantize")
        self.timers = {k: KernelTimer(t) for k in keys}
        self.host_in = t.from_numpy(bits.view(np.int16)).view(t.bfloat16).pin_memory()
        self.dev_in = t.empty_like(self.x[0])

    def single_kernel(self):
        if self.fused_deq:
            return ("amax+quantize_dequantize_rtn", "quantize_dequantize_sr")
        return ("quantize_sr", "dequantize")

    def step(self, i, timed=False, x=None):
        F = self.F
        x = self.x[i % self.n_inputs] if x is None else x
        T = self.timers if timed else None

        def run(key, fn):
            return T[key].around(fn) if T is not None else fn()

        if self.fused_deq:
            run("amax+quantize_dequantize_rtn", lambda: F.fp4_quantize_dequantize(
                x, fmt=self.fmt, rnd="rtn", codes=self.codes[0], scales=self.scales[0], tensor_scale_out=self.ts,
                out=self.deq[0]))
            run("quantize_dequantize_sr", lambda: F.fp4_quantize_dequantize(
                x, fmt=self.fmt, rnd="sr", seed=1, tensor_scale_in=self.ts, codes=self.codes[1],
                scales=self.scales[1], tensor_scale_out=self.ts_sr, out=self.deq[1]))
            return

        # RTN: tensor amax + quantize (one entry point), then dequantize
        run("amax+quantize_rtn", lambda: F.fp4_quantize(x, fmt=self.fmt, rnd="rtn", codes=self.codes[0],
                                                   scales=self.scales[0], tensor_scale_out=self.ts))
        run("dequantize", lambda: F.fp4_dequantize(self.codes[0], self.scales[0], self.ts, fmt="nvfp4",
                                                   out=self.deq[0]))
        # SR with the same tensor scale, then dequantize
        run("quantize_sr", lambda: F.fp4_quantize(x, fmt=self.fmt, rnd="sr", seed=1, tensor_scale_in=self.ts,
                                                  codes=self.codes[1], scales=self.scales[1],
                                                  tensor_scale_out=self.ts_sr))
        run("dequantize", lambda: F.fp4_dequantize(self.codes[1], self.scales[1], self.ts_sr, fmt="nvfp4",
                                                   out=self.deq[1]))

    def outputs(self):
        return [self.codes[0], self.scales[0], self.ts, self.deq[0], self.codes[1], self.scales[1], self.ts_sr,
                self.deq[1]]

    def e2e_step(self, host_outs):
        self.dev_in.copy_(self.host_in, non_blocking=True)
        self.step(0, x=self.dev_in)
        for h, o in zip(host_outs, self.outputs()):
            h.copy_(o, non_blocking=True)
        return (self.host_in.numel() * self.host_in.element_size(),
                sum(o.numel() * o.element_size() for o in self.outputs()))

    def family_work(self, key):
        """Algorithmic work per step of a kernel family (bytes here)."""
        return {"amax+quantize_rtn": self.q_bytes, "quantize_sr": self.q_bytes, "dequantize": 2 * self.d_bytes,
                "amax+quantize_dequantize_rtn": self.q_bytes + self.d_bytes,
                "quantize_dequantize_sr": self.q_bytes + self.d_bytes}[key]

    def family_launches(self, key):
        """Launches of a kernel family per step."""
        return 2 if key == "dequantize" else 1

    def solo_calls(self):
        """Each kernel family's launch alone (for _solo_times): key -> (call(i), launches per step)."""
        if not self.fused_deq:
            return None
        F = self.F
        return {
            "amax+quantize_dequantize_rtn": (lambda i: F.fp4_quantize_dequantize(
                self.x[i % self.n_inputs], fmt=self.fmt, rnd="rtn", codes=self.codes[0], scales=self.scales[0],
                tensor_scale_out=self.ts, out=self.deq[0]), 1),
            "quantize_dequantize_sr": (lambda i: F.fp4_quantize_dequantize(
                self.x[i % self.n_inputs], fmt=self.fmt, rnd="sr", seed=1, tensor_scale_in=self.ts,
                codes=self.codes[1], scales=self.scales[1], tensor_scale_out=self.ts_sr, out=self.deq[1]), 1),
        }

    def family_elements(self, key):
        """Elements a kernel family processes per step (each launch covers the whole tensor)."""
        return self.n * self.family_launches(key)

    def value_from_ms(self, ms_per_step, n_ranks):
        return self.step_bytes * n_ranks / (ms_per_step * 1e-3) / 1e9

    def config(self):
        return {"workload": self.name, "shape": [self.rows, self.cols], "format": self.fmt, "block": 16,
                "distribution": "0.1*student_t(3)", "seed": 1, "rounding": ["rtn", "sr(philox4x32-10, seed 1)"],
                "dequantize": "f32, in the quantizing launch" if self.fused_deq else "f32, separate launch",
                "algorithmic_bytes_per_step": self.step_bytes,
                "l2": f"{self.n_inputs} rotating input copies (128 MB) and ~146 MB written per step"}

    # ---- CPU oracle on the same workload ----
    def oracle_setup(self):
        from workloads import nvfp4_student_t
        self.host_bits = nvfp4_student_t(self.rows, self.cols, seed=1)

    def oracle_step(self, rows):
        import oracle as O
        from workloads import bf16_to_f32
        x32 = bf16_to_f32(self.host_bits[:rows]) if rows < self.rows else bf16_to_f32(self.host_bits)
        s_t = O.nv_tensor_scale(bf16_to_f32(self.host_bits))
        r = O.quantize_values(x32, fmt=self.fmt, rnd="rtn", tensor_scale=s_t)
        O.dequantize(r["codes"], r["scales"], fmt="nvfp4", tensor_scale=s_t)
        r = O.quantize_values(x32, fmt=self.fmt, rnd="sr", seed=1, tensor_scale=s_t)
        O.dequantize(r["codes"], r["scales"], fmt="nvfp4", tensor_scale=s_t)
        return rows * self.cols * self.step_bytes / self.n

    def cpu_sample(self):
        return self.rows, f"one full step ({self.rows}x{self.cols}) on the host, NumPy elementwise (1 thread)"

    def reference_sample(self):
        return 256, f"256 of {self.rows} rows per step (global tensor scale), NumPy 1 thread"


class NvfpStudentT46(NvfpStudentT):
    """The same step with four-over-six block scales (per block the lower-error of max->6 and
    max->4); its codes and scales are NVFP4, dequantized as such."""

    name = "nvfp4_4o6_student_t_4096"
    fmt = "nvfp4_4o6"
    fused_deq = False            # four-over-six quantizes, then a separate dequantize launch
    launches_per_step = 4
    gemm_companion = False

    def cpu_sample(self):
        return 512, f"512 of {self.rows} rows (global tensor scale), NumPy elementwise (1 thread)"

    def reference_sample(self):
        return 64, f"64 of {self.rows} rows per step (global tensor scale), NumPy 1 thread"


class Nvfp2dWeight(Workload):
    """Square-tile (16x16) NVFP4 quantization of a Llama MLP weight W[11008, 4096] ~ N(0, 0.02), RTN:
    W's codes along K and W^T's codes along N from one rounding, one scale per tile."""

    name = "nvfp4_2d_weight_11008x4096"
    rows, cols = 11008, 4096
    n_inputs = 2                 # two rotating weight copies (180 MB > L2)
    launches_per_step = 3        # tensor amax, s_t = amax / 2688, 2-D quantize
    unit = "GB/s"

    def __init__(self, torch, F):
        self.t, self.F = torch, F
        n = self.rows * self.cols
        # bf16 in; codes and E4M3 scales out twice (W and W^T); the amax pass is a second read of W
        self.step_bytes = n * (2 + 2 * (0.5 + 1 / 16))
        self.amax_bytes = n * 2.0

    def _bits(self):
        from workloads import normal_bf16
        return normal_bf16((self.rows, self.cols), 0.02, 11, 0)

    def setup(self, device):
        t = self.t
        bits = self._bits()
        self.host_in = _pinned_bf16(t, bits)
        self.x = [self.host_in.to(device).clone() for _ in range(self.n_inputs)]
        self.dev_in = t.empty_like(self.x[0])
        q, qt = self.F.fp4_quantize_2d(self.x[0], fmt="nvfp4", sf_layout="mma")
        self.q, self.qt = q, qt
        self.amax = t.empty((1,), dtype=t.float32, device=device)
        self.timers = {k: KernelTimer(t) for k in ("amax", "quantize_2d")}

    def single_kernel(self):
        return ("quantize_2d",)

    def step(self, i, timed=False, x=None):
        F = self.F
        x = self.x[i % self.n_inputs] if x is None else x
        T = self.timers if timed else None

        def run(key, fn):
            return T[key].around(fn) if T is not None else fn()

        def amax():
            F.fp4_amax(x, out=self.amax)
            F.fp4_nv_tensor_scale(self.amax, out=self.q.tensor_scale)

        run("amax", amax)
        run("quantize_2d", lambda: F.fp4_quantize_2d(
            x, fmt="nvfp4", sf_layout="mma", tensor_scale_in=self.q.tensor_scale, codes=self.q.codes,
            scales=self.q.scales, codes_t=self.qt.codes, scales_t=self.qt.scales,
            tensor_scale_out=self.q.tensor_scale))

    def outputs(self):
        return [self.q.codes, self.q.scales, self.qt.codes, self.qt.scales, self.q.tensor_scale]

    def e2e_step(self, host_outs):
        self.dev_in.copy_(self.host_in, non_blocking=True)
        self.step(0, x=self.dev_in)
        for h, o in zip(host_outs, self.outputs()):
            h.copy_(o, non_blocking=True)
        return (self.host_in.numel() * 2, sum(o.numel() * o.element_size() for o in self.outputs()))

    def family_work(self, key):
        return {"amax": self.amax_bytes, "quantize_2d": self.step_bytes}[key]

    def value_from_ms(self, ms_per_step, n_ranks):
        return self.step_bytes * n_ranks / (ms_per_step * 1e-3) / 1e9

    def config(self):
        return {"workload": self.name, "shape": [self.rows, self.cols], "format": "nvfp4", "block": "16x16",
                "distribution": "normal(0, 0.02)", "seed": 11, "rounding": "rtn", "outputs": "W and W^T",
                "sf_layout": "mma", "algorithmic_bytes_per_step": self.step_bytes,
                "l2": f"{self.n_inputs} rotating weight copies (180 MB)"}

    def oracle_setup(self):
        self.host_bits = self._bits()

    def oracle_step(self, rows):
        import oracle as O
        from workloads import bf16_to_f32
        s_t = O.nv_tensor_scale(bf16_to_f32(self.host_bits))
        O.quantize_2d(self.host_bits[:rows], fmt="nvfp4", tensor_scale=s_t)
        return rows * self.cols * (2 + 2 * (0.5 + 1 / 16))

    def cpu_sample(self):
        return 2048, f"2048 of {self.rows} rows (global tensor scale), NumPy (1 thread)"

    def reference_sample(self):
        return 512, f"512 of {self.rows} rows per step (global tensor scale), NumPy 1 thread"


class NvfpMseWeight(Workload):
    """NVFP4 quantization of a Llama MLP weight W[11008, 4096] ~ N(0, 0.02) with MSE-searched scales:
    one tensor step (17 tensor scales, each with a 17-byte block step) and the final block step, RTN.
    Bound by instruction issue, so its roofline counts candidate evaluations (one element quantized,
    dequantized and its squared error accumulated under one candidate scale)."""

    name = "nvfp4_mse_weight_11008x4096"
    rows, cols = 11008, 4096
    iters = 1
    n_inputs = 2
    launches_per_step = 3        # amax, tensor step, block step + codes
    unit = "GB/s"
    evals_per_element = 17 * 17 * 1 + 17       # tensor step(s) + final block step
    instr_per_eval = 5           # quotient multiply, 1/2 E2M1 conversion, 1/2 back + widen, subtract, fma

    def __init__(self, torch, F):
        self.t, self.F = torch, F
        n = self.rows * self.cols
        self.n = n
        self.step_bytes = n * (2 + 0.5 + 1 / 16)

    def _bits(self):
        from workloads import normal_bf16
        return normal_bf16((self.rows, self.cols), 0.02, 12, 0)

    def setup(self, device):
        t = self.t
        self.host_in = _pinned_bf16(t, self._bits())
        self.x = [self.host_in.to(device).clone() for _ in range(self.n_inputs)]
        self.dev_in = t.empty_like(self.x[0])
        self.q = self.F.fp4_quantize_mse(self.x[0], iters=self.iters, sf_layout="mma")
        self.timers = {"quantize_mse": KernelTimer(t)}

    def single_kernel(self):
        return ("quantize_mse",)

    def family_bound(self, key):
        return "alu"

    def alu_peak(self, sms):
        return sms * 128 * 1.965e9 / self.instr_per_eval, self.instr_per_eval

    def step(self, i, timed=False, x=None):
        x = self.x[i % self.n_inputs] if x is None else x
        fn = lambda: self.F.fp4_quantize_mse(x, iters=self.iters, sf_layout="mma", codes=self.q.codes,
                                             scales=self.q.scales, tensor_scale_out=self.q.tensor_scale)
        return self.timers["quantize_mse"].around(fn) if timed else fn()

    def outputs(self):
        return [self.q.codes, self.q.scales, self.q.tensor_scale]

    def e2e_step(self, host_outs):
        self.dev_in.copy_(self.host_in, non_blocking=True)
        self.step(0, x=self.dev_in)
        for h, o in zip(host_outs, self.outputs()):
            h.copy_(o, non_blocking=True)
        return (self.host_in.numel() * 2, sum(o.numel() * o.element_size() for o in self.outputs()))

    def family_work(self, key):
        return self.n * self.evals_per_element

    def value_from_ms(self, ms_per_step, n_ranks):
        return self.step_bytes * n_ranks / (ms_per_step * 1e-3) / 1e9

    def config(self):
        return {"workload": self.name, "shape": [self.rows, self.cols], "format": "nvfp4", "block": 16,
                "distribution": "normal(0, 0.02)", "seed": 12, "rounding": "rtn", "tensor_steps": self.iters,
                "sf_layout": "mma", "algorithmic_bytes_per_step": self.step_bytes,
                "candidate_evaluations_per_step": self.n * self.evals_per_element,
                "l2": f"{self.n_inputs} rotating weight copies (180 MB)"}

    def oracle_setup(self):
        self.host_bits = self._bits()

    def oracle_step(self, rows):
        import oracle as O
        O.quantize_mse(self.host_bits[:rows], iters=self.iters)
        return rows * self.cols * (2 + 0.5 + 1 / 16)

    def cpu_sample(self):
        return 32, f"32 of {self.rows} rows searched on their own (tensor scale of the sample), NumPy (1 thread)"

    def reference_sample(self):
        return 8, f"8 of {self.rows} rows per step searched on their own, NumPy 1 thread"


def _dev_bf16(torch, bits, device):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def _pinned_bf16(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


class GemmWorkload(Workload):
    """Common parts of the quantize + block-scaled GEMM workloads (value in TFLOP/s of GEMM work)."""

    unit = "TFLOP/s"

    def family_bound(self, key):
        return "tensor" if key == "gemm" else "hbm"

    def value_from_ms(self, ms_per_step, n_ranks):
        return self.step_flops * n_ranks / (ms_per_step * 1e-3) / 1e12

    def outputs(self):
        return self.outs


class HadamardMxGemm(GemmWorkload):
    """Block-Hadamard-rotated MXFP4 quantize of X[8192,4096] (1% channels x50) fused with the GEMM
    against W[11008,4096] (rotated and quantized offline), bf16 out, for b = 16, 32, 64, 128."""

    name = "hadamard_mxfp4_gemm_8192x11008x4096"
    M, N, K = 8192, 11008, 4096
    blocks = (16, 32, 64, 128)
    launches_per_step = 8

    def __init__(self, torch, F):
        self.t, self.F = torch, F
        self.gemm_flops = 2.0 * self.M * self.N * self.K
        self.step_flops = len(self.blocks) * self.gemm_flops
        self.q_bytes = self.M * self.K * (2 + 0.5 + 1 / 32)

    def setup(self, device):
        from workloads import hadamard_acts, hadamard_weights
        t, F = self.t, self.F
        self.host_bits = hadamard_acts(self.M, self.K, seed=2)
        wb = hadamard_weights(self.N, self.K, seed=2)
        self.x = _dev_bf16(t, self.host_bits, device)
        w = _dev_bf16(t, wb, device)
        self.qw = {b: F.fp4_hadamard_quantize(w, b, fmt="mxfp4", sf_layout="mma") for b in self.blocks}
        del w
        self.codes = t.empty((self.M, self.K // 2), dtype=t.uint8, device=device)
        self.scales = t.empty((F.fp4_scales_bytes(self.M, self.K, 32, 1, "mma"),), dtype=t.uint8, device=device)
        self.outs = [t.empty((self.M, self.N), dtype=t.bfloat16, device=device) for _ in self.blocks]
        self.timers = {k: KernelTimer(t) for k in ("rotate_quantize", "gemm")}
        self.host_in = _pinned_bf16(t, self.host_bits)
        self.dev_in = t.empty_like(self.x)

    def single_kernel(self):
        return ("rotate_quantize", "gemm")

    def solo_calls(self):
        """Each family alone (for _solo_times): rotate+quantize over three input copies (192 MB, past
        L2), the GEMMs writing their 180 MB outputs; every block size in turn."""
        F, nb = self.F, len(self.blocks)
        if not hasattr(self, "x_copies"):
            self.x_copies = [self.x] + [self.x.clone() for _ in range(2)]

        def rq(i):
            b = self.blocks[i % nb]
            F.fp4_hadamard_quantize(self.x_copies[i % 3], b, fmt="mxfp4", sf_layout="mma", codes=self.codes,
                                    scales=self.scales)

        def gm(i):
            qw = self.qw[self.blocks[i % nb]]
            F.fp4_gemm(self.codes, self.scales, qw.codes, qw.scales, fmt="mxfp4", out_dtype="bf16",
                       out=self.outs[i % nb])

        return {"rotate_quantize": (rq, nb), "gemm": (gm, nb)}

    def step(self, i, timed=False, x=None):
        F = self.F
        x = self.x if x is None else x
        T = self.timers if timed else None

        def run(key, fn):
            return T[key].around(fn) if T is not None else fn()

        for b, y in zip(self.blocks, self.outs):
            run("rotate_quantize", lambda: F.fp4_hadamard_quantize(x, b, fmt="mxfp4", sf_layout="mma",
                                                                   codes=self.codes, scales=self.scales))
            qw = self.qw[b]
            run("gemm", lambda: F.fp4_gemm(self.codes, self.scales, qw.codes, qw.scales, fmt="mxfp4",
                                           out_dtype="bf16", out=y))

    def e2e_step(self, host_outs):
        self.dev_in.copy_(self.host_in, non_blocking=True)
        self.step(0, x=self.dev_in)
        for h, o in zip(host_outs, self.outs):
            h.copy_(o, non_blocking=True)
        return (self.host_in.numel() * 2, sum(o.numel() * 2 for o in self.outs))

    def family_work(self, key):
        return len(self.blocks) * (self.q_bytes if key == "rotate_quantize" else self.gemm_flops)

    def config(self):
        return {"workload": self.name, "M": self.M, "N": self.N, "K": self.K, "format": "mxfp4", "block": 32,
                "hadamard_blocks": list(self.blocks), "activations": "N(0,1), 41 of 4096 channels x50, seed 2",
                "weights": "N(0,0.02), rotated and quantized offline (untimed)", "out": "bf16",
                "gemm_flops_per_step": self.step_flops,
                "l2": f"inputs + {len(self.blocks)} x 180 MB bf16 outputs per step exceed L2"}

    def oracle_setup(self):
        from workloads import hadamard_acts, hadamard_weights
        import oracle as O
        self.host_bits = hadamard_acts(self.M, self.K, seed=2)
        self.ow = O.quantize(hadamard_weights(self.N, self.K, seed=2)[:256], fmt="mxfp4", had_block=128)

    def oracle_step(self, rows):
        import oracle as O
        qx = O.quantize(self.host_bits[:rows], fmt="mxfp4", had_block=128)
        O.gemm_ref(qx, self.ow, "mxfp4")
        return 2.0 * rows * 256 * self.K

    def cpu_sample(self):
        return 64, "b = 128: rotate+quantize 64 rows of X and their fp64 GEMM against 256 rows of W (NumPy)"

    def reference_sample(self):
        return 16, "b = 128: rotate+quantize 16 rows of X and their fp64 GEMM against 256 rows of W (NumPy)"


class HadamardMxGemm128(HadamardMxGemm):
    """The Hadamard workload at one block size, b = 128: one rotate+quantize of X[8192,4096] and one
    GEMM against W[11008,4096] per step.  The default workload's line carries it as the GEMM half of
    the metric."""

    name = "hadamard_mxfp4_gemm_8192x11008x4096_b128"
    blocks = (128,)
    launches_per_step = 2

    def release(self):
        for a in ("x", "x_copies", "qw", "codes", "scales", "outs", "host_in", "dev_in"):
            if hasattr(self, a):
                delattr(self, a)


class FusedMxLinear(GemmWorkload):
    """One MXFP4 linear of an FP4 pipeline: Y = X W^T with X[8192,4096] ~ N(0,1) and W[11008,4096] ~
    N(0,0.02) as resident MXFP4 operands, whose epilogue quantizes Y (RTN, MXFP4) into the next
    layer's codes and tensor-core-layout scales; Y itself is never written."""

    name = "mxfp4_fused_linear_8192x11008x4096"
    M, N, K = 8192, 11008, 4096
    launches_per_step = 1

    def __init__(self, torch, F):
        self.t, self.F = torch, F
        self.step_flops = 2.0 * self.M * self.N * self.K

    def setup(self, device):
        from workloads import normal_bf16
        t, F = self.t, self.F
        xb, wb = normal_bf16((self.M, self.K), 1.0, 13, 0), normal_bf16((self.N, self.K), 0.02, 13, 1)
        self.host_in = (_pinned_bf16(t, xb), _pinned_bf16(t, wb))
        self.dev_in = tuple(t.empty_like(h, device=device) for h in self.host_in)
        self.qx = F.fp4_quantize(self.host_in[0].to(device), fmt="mxfp4", sf_layout="mma")
        self.qw = F.fp4_quantize(self.host_in[1].to(device), fmt="mxfp4", sf_layout="mma")
        self.codes = t.empty((self.M, self.N // 2), dtype=t.uint8, device=device)
        self.scales = t.empty((F.fp4_scales_bytes(self.M, self.N, 32, 1, "mma"),), dtype=t.uint8, device=device)
        self.outs = [self.codes, self.scales]
        self.timers = {"gemm_quantize": KernelTimer(t), "quantize": KernelTimer(t)}

    def single_kernel(self):
        return ("gemm_quantize",)

    def family_bound(self, key):
        return "tensor" if key == "gemm_quantize" else "hbm"

    def step(self, i, timed=False, q=None):
        F = self.F
        qx, qw = (self.qx, self.qw) if q is None else q
        fn = lambda: F.fp4_gemm_quantize(qx.codes, qx.scales, qw.codes, qw.scales, fmt="mxfp4", out_fmt="mxfp4",
                                         codes=self.codes, scales=self.scales)
        return self.timers["gemm_quantize"].around(fn) if timed else fn()

    def e2e_step(self, host_outs):
        # end to end: bf16 X and W from pinned host memory, both quantized, the fused linear, codes
        # and scales back
        F = self.F
        for h, d in zip(self.host_in, self.dev_in):
            d.copy_(h, non_blocking=True)
        qx = F.fp4_quantize(self.dev_in[0], fmt="mxfp4", sf_layout="mma", codes=self.qx.codes, scales=self.qx.scales)
        qw = F.fp4_quantize(self.dev_in[1], fmt="mxfp4", sf_layout="mma", codes=self.qw.codes, scales=self.qw.scales)
        self.step(0, q=(qx, qw))
        for h, o in zip(host_outs, self.outs):
            h.copy_(o, non_blocking=True)
        return (sum(h.numel() * 2 for h in self.host_in), sum(o.numel() for o in self.outs))

    def family_work(self, key):
        return self.step_flops

    def config(self):
        return {"workload": self.name, "M": self.M, "N": self.N, "K": self.K, "format": "mxfp4", "block": 32,
                "activations": "N(0,1), seed 13", "weights": "N(0,0.02), quantized offline (untimed)",
                "out": "MXFP4 codes + scales of Y (RTN, tensor-core layout), Y not written",
                "gemm_flops_per_step": self.step_flops, "l2": "operands 69 MB + 48 MB of output codes per step"}

    def oracle_setup(self):
        from workloads import normal_bf16
        import oracle as O
        self.xb = normal_bf16((self.M, self.K), 1.0, 13, 0)
        self.ow = O.quantize(normal_bf16((self.N, self.K), 0.02, 13, 1)[:1024], fmt="mxfp4")

    def oracle_step(self, rows):
        import oracle as O
        qx = O.quantize(self.xb[:rows], fmt="mxfp4")
        y, _ = O.gemm_ref(qx, self.ow, "mxfp4")
        O.quantize_values(y.astype(np.float32), fmt="mxfp4")
        return 2.0 * rows * 1024 * self.K

    def cpu_sample(self):
        return 8192, "all 8192 rows of X: quantize, fp64 GEMM against 1024 rows of W, quantize the product (NumPy)"

    def reference_sample(self):
        return 64, "64 rows of X: quantize, fp64 GEMM against 1024 rows of W, quantize the product (NumPy)"


class VitLinears(GemmWorkload):
    """ViT-B/16 training linears at M = 256*197 = 50432: per layer (qkv, fc1, fc2) the forward
    (RTN), dgrad and wgrad GEMMs, each operand quantized to MXFP4 along its own contraction axis
    (dY with Philox SR, seeds 3 and 4), bf16 outputs."""

    name = "vit_b16_linears_50432"
    layers = ("qkv", "fc1", "fc2")
    launches_per_step = 27
    M = 256 * 197

    def __init__(self, torch, F):
        self.t, self.F = torch, F
        from workloads import VIT_LAYERS
        self.dims = {l: VIT_LAYERS[l] for l in self.layers}        # (K, N)
        self.step_flops = sum(3 * 2.0 * self.M * k * n for k, n in self.dims.values())
        per = 2 + 0.5 + 1 / 32
        self.q_bytes = {"quantize": sum(self.M * k + n * k + self.M * n for k, n in self.dims.values()) * per,
                        "quantize_axis0": sum(n * k + self.M * n + self.M * k for k, n in self.dims.values()) * per}

    def setup(self, device):
        from workloads import vit_layer
        t = self.t
        self.host = {}
        self.dev = {}
        for l in self.layers:
            xb, wb, dyb = vit_layer(l)
            self.host[l] = (_pinned_bf16(t, xb), _pinned_bf16(t, wb), _pinned_bf16(t, dyb))
            self.dev[l] = tuple(h.to(device) for h in self.host[l])
        self.outs = []
        for l in self.layers:
            k, n = self.dims[l]
            self.outs += [t.empty((self.M, n), dtype=t.bfloat16, device=device),
                          t.empty((self.M, k), dtype=t.bfloat16, device=device),
                          t.empty((n, k), dtype=t.bfloat16, device=device)]
        self.timers = {k: KernelTimer(t) for k in ("quantize", "quantize_axis0", "gemm")}
        self.dev_in = {l: tuple(t.empty_like(d) for d in self.dev[l]) for l in self.layers}

    def single_kernel(self):
        return ("quantize", "quantize_axis0", "gemm")

    def step(self, i, timed=False, use_e2e_inputs=False):
        F = self.F
        T = self.timers if timed else None

        def run(key, fn):
            return T[key].around(fn) if T is not None else fn()

        def q(key, x, axis, rnd="rtn", seed=0):
            return run(key, lambda: F.fp4_quantize(x, fmt="mxfp4", axis=axis, rnd=rnd, seed=seed, sf_layout="mma"))

        for li, l in enumerate(self.layers):
            x, w, dy = (self.dev_in if use_e2e_inputs else self.dev)[l]
            y, dx, dw = self.outs[3 * li:3 * li + 3]
            qx, qw = q("quantize", x, 1), q("quantize", w, 1)
            run("gemm", lambda: F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="mxfp4",
                                           out_dtype="bf16", out=y))
            qdy, qwt = q("quantize", dy, 1, "sr", 3), q("quantize_axis0", w, 0)
            run("gemm", lambda: F.fp4_gemm(qdy.codes, qdy.scales, qwt.codes, qwt.scales, fmt="mxfp4",
                                           out_dtype="bf16", out=dx))
            qdyt, qxt = q("quantize_axis0", dy, 0, "sr", 4), q("quantize_axis0", x, 0)
            run("gemm", lambda: F.fp4_gemm(qdyt.codes, qdyt.scales, qxt.codes, qxt.scales, fmt="mxfp4",
                                           out_dtype="bf16", out=dw))

    def e2e_step(self, host_outs):
        h2d = 0
        for l in self.layers:
            for h, d in zip(self.host[l], self.dev_in[l]):
                d.copy_(h, non_blocking=True)
                h2d += h.numel() * 2
        self.step(0, use_e2e_inputs=True)
        for h, o in zip(host_outs, self.outs):
            h.copy_(o, non_blocking=True)
        return h2d, sum(o.numel() * 2 for o in self.outs)

    def family_work(self, key):
        return self.step_flops if key == "gemm" else self.q_bytes[key]

    def config(self):
        return {"workload": self.name, "M": self.M, "layers": {l: {"K": k, "N": n} for l, (k, n) in self.dims.items()},
                "format": "mxfp4", "block": 32, "passes": ["fwd (RTN)", "dgrad (dY SR seed 3, W axis 0)",
                                                          "wgrad (dY axis 0 SR seed 4, X axis 0)"],
                "out": "bf16", "gemm_flops_per_step": self.step_flops,
                "l2": "~1.5 GB of operands and outputs per step exceed L2"}

    def oracle_setup(self):
        from workloads import vit_layer
        import oracle as O
        self.xb, wb, _ = vit_layer("fc1")
        self.ow = O.quantize(wb[:256], fmt="mxfp4")

    def oracle_step(self, rows):
        import oracle as O
        qx = O.quantize(self.xb[:rows], fmt="mxfp4")
        O.gemm_ref(qx, self.ow, "mxfp4")
        return 2.0 * rows * 256 * self.xb.shape[1]

    def cpu_sample(self):
        return 256, "fc1 forward: quantize 256 rows of X and their fp64 GEMM against 256 rows of W (NumPy)"

    def reference_sample(self):
        return 64, "fc1 forward: quantize 64 rows of X and their fp64 GEMM against 256 rows of W (NumPy)"


class LlamaNvfp4(GemmWorkload):
    """Llama-7B-shaped NVFP4 sweep: for (K, N) in {(4096, 4096), (4096, 11008), (11008, 4096)} and
    M in {1, 16, 128, 1024, 4096, 16384}: tensor amax + quantize X[:M] (0.5% channels x20) and
    the GEMM against W (quantized offline), bf16 out, timed end to end per case."""

    name = "llama7b_nvfp4_sweep"
    shapes = ((4096, 4096), (4096, 11008), (11008, 4096))
    Ms = (1, 16, 128, 1024, 4096, 16384)
    bracket = False
    flush_between_cases = True
    launches_per_step = 36

    def __init__(self, torch, F):
        self.t, self.F = torch, F
        self.cases = [(k, n, m) for k, n in self.shapes for m in self.Ms]
        self.step_flops = sum(2.0 * m * n * k for k, n, m in self.cases)

    def setup(self, device):
        from workloads import llama_acts, llama_weights
        t, F = self.t, self.F
        self.host_x = {k: _pinned_bf16(t, llama_acts(k, 16384, seed=4)) for k in (4096, 11008)}
        self.x = {k: h.to(device) for k, h in self.host_x.items()}
        self.qw = {}
        for k, n in self.shapes:
            w = _dev_bf16(t, llama_weights(k, n, seed=4), device)
            self.qw[(k, n)] = F.fp4_quantize(w, fmt="nvfp4", sf_layout="mma")
            del w
        self.outs = [t.empty((m, n), dtype=t.bfloat16, device=device) for k, n, m in self.cases]
        self.timers = {k: KernelTimer(t) for k in ("amax+quantize", "gemm")}
        self.case_timers = [KernelTimer(t) for _ in self.cases]
        self.flush = t.zeros((64 * 1024 * 1024,), dtype=t.int32, device=device)
        self.dev_in = {k: t.empty_like(v) for k, v in self.x.items()}

    def single_kernel(self):
        return ("gemm",)

    def _case(self, ci, x, timed):
        F = self.F
        k, n, m = self.cases[ci]
        qw, y = self.qw[(k, n)], self.outs[ci]
        xm = x[k][:m]
        if not timed:
            qx = F.fp4_quantize(xm, fmt="nvfp4", sf_layout="mma")
            F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="nvfp4", a_tensor_scale=qx.tensor_scale,
                       b_tensor_scale=qw.tensor_scale, out_dtype="bf16", out=y)
            return
        t = self.t
        e = [t.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        qx = F.fp4_quantize(xm, fmt="nvfp4", sf_layout="mma")
        e[1].record()
        F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="nvfp4", a_tensor_scale=qx.tensor_scale,
                   b_tensor_scale=qw.tensor_scale, out_dtype="bf16", out=y)
        e[2].record()
        self.timers["amax+quantize"].pairs.append((e[0], e[1]))
        self.timers["gemm"].pairs.append((e[1], e[2]))
        self.case_timers[ci].pairs.append((e[0], e[2]))

    def step(self, i, timed=False, use_e2e_inputs=False):
        x = self.dev_in if use_e2e_inputs else self.x
        if timed:
            # ~2 ms of GPU sleep (untimed) while the host enqueues the step's 18 cases, so that no
            # case's events also measure the host's launch latency
            self.t.cuda._sleep(4_000_000)
        for ci in range(len(self.cases)):
            if self.flush_between_cases:
                self.flush.max()                 # between timed cases: a 256 MB read evicts the previous case from L2
            self._case(ci, x, timed)

    def timed_ms_total(self):
        return sum(sum(a.elapsed_time(b) for a, b in ct.pairs) for ct in self.case_timers)

    def e2e_step(self, host_outs):
        h2d = 0
        for k, h in self.host_x.items():
            self.dev_in[k].copy_(h, non_blocking=True)
            h2d += h.numel() * 2
        self.step(0, use_e2e_inputs=True)
        for h, o in zip(host_outs, self.outs):
            h.copy_(o, non_blocking=True)
        return h2d, sum(o.numel() * 2 for o in self.outs)

    def family_work(self, key):
        if key == "gemm":
            return self.step_flops
        return sum(m * k * (2 + 0.5 + 1 / 16) for k, n, m in self.cases)

    def cases_summary(self, steps):
        out = {}
        for (k, n, m), ct in zip(self.cases, self.case_timers):
            ms = float(np.mean([a.elapsed_time(b) for a, b in ct.pairs]))
            wgb = n * k * (0.5 + 1 / 16) / (ms * 1e-3) / 1e9          # weight codes + E4M3 scales streamed
            out[f"K{k}_N{n}_M{m}"] = {"us": round(ms * 1e3, 2), "tflops": round(2.0 * m * n * k / (ms * 1e-3) / 1e12, 1),
                                      "weight_gbs": round(wgb, 1)}
        return out

    def config(self):
        return {"workload": self.name, "shapes_KN": [list(s) for s in self.shapes], "M": list(self.Ms),
                "format": "nvfp4", "block": 16, "activations": "N(0,1), 0.5% channels x20, seed 4",
                "weights": "N(0,0.02), quantized offline (untimed)", "out": "bf16",
                "gemm_flops_per_step": self.step_flops,
                "l2": "256 MB read between cases (untimed) and a GPU sleep while the host enqueues a step; "
                      "ms_per_step sums the per-case event times"}

    def oracle_setup(self):
        from workloads import llama_acts, llama_weights
        import oracle as O
        from workloads import bf16_to_f32
        self.xb = llama_acts(4096, 4096, seed=4)
        self.s_t = O.nv_tensor_scale(bf16_to_f32(self.xb))
        self.ow = O.quantize(llama_weights(4096, 4096, seed=4)[:256], fmt="nvfp4")

    def oracle_step(self, rows):
        import oracle as O
        qx = O.quantize(self.xb[:rows], fmt="nvfp4", tensor_scale=self.s_t)
        O.gemm_ref(qx, self.ow, "nvfp4")
        return 2.0 * rows * 256 * 4096

    def cpu_sample(self):
        return 128, "K = N = 4096, M = 4096: quantize 128 rows of X and their fp64 GEMM against 256 rows of W (NumPy)"

    def reference_sample(self):
        return 32, "K = N = 4096, M = 4096: quantize 32 rows of X and their fp64 GEMM against 256 rows of W (NumPy)"


class MxLinear128(GemmWorkload):
    """MXFP4 quantized linear forward: X[128,512] ~ N(0,1), W[512,512] ~ N(0,0.02), RTN, fp32 out."""

    name = "mx_linear_128x512"
    M, N, K = 128, 512, 512
    launches_per_step = 3

    def __init__(self, torch, F):
        self.t, self.F = torch, F
        self.step_flops = 2.0 * self.M * self.N * self.K

    def setup(self, device):
        from workloads import mx_linear_128x512
        t = self.t
        xb, wb = mx_linear_128x512(0)
        self.host = (_pinned_bf16(t, xb), _pinned_bf16(t, wb))
        self.x, self.w = (h.to(device) for h in self.host)
        self.dev_in = tuple(t.empty_like(h, device=device) for h in self.host)
        self.outs = [t.empty((self.M, self.N), dtype=t.float32, device=device)]
        self.timers = {k: KernelTimer(t) for k in ("quantize", "gemm")}

    def single_kernel(self):
        return ("gemm",)

    def step(self, i, timed=False, use_e2e_inputs=False):
        F = self.F
        T = self.timers if timed else None
        x, w = self.dev_in if use_e2e_inputs else (self.x, self.w)

        def run(key, fn):
            return T[key].around(fn) if T is not None else fn()

        qx = run("quantize", lambda: F.fp4_quantize(x, fmt="mxfp4", sf_layout="mma"))
        qw = run("quantize", lambda: F.fp4_quantize(w, fmt="mxfp4", sf_layout="mma"))
        run("gemm", lambda: F.fp4_gemm(qx.codes, qx.scales, qw.codes, qw.scales, fmt="mxfp4", out_dtype="f32",
                                       out=self.outs[0]))

    def e2e_step(self, host_outs):
        for h, d in zip(self.host, self.dev_in):
            d.copy_(h, non_blocking=True)
        self.step(0, use_e2e_inputs=True)
        host_outs[0].copy_(self.outs[0], non_blocking=True)
        return sum(h.numel() * 2 for h in self.host), self.outs[0].numel() * 4

    def family_work(self, key):
        return self.step_flops if key == "gemm" else (self.M + self.N) * self.K * (2 + 0.5 + 1 / 32)

    def config(self):
        return {"workload": self.name, "M": self.M, "N": self.N, "K": self.K, "format": "mxfp4", "block": 32,
                "seed": 0, "out": "f32", "l2": "latency-bound (0.4 MB of operands, L2-resident)"}

    def oracle_setup(self):
        from workloads import mx_linear_128x512
        self.xb, self.wb = mx_linear_128x512(0)

    def oracle_step(self, rows):
        import oracle as O
        qx = O.quantize(self.xb[:rows], fmt="mxfp4")
        qw = O.quantize(self.wb, fmt="mxfp4")
        O.gemm_ref(qx, qw, "mxfp4")
        return 2.0 * rows * self.N * self.K

    def cpu_sample(self):
        return 128, "the whole workload: quantize X and W, fp64 GEMM (NumPy)"

    def reference_sample(self):
        return 128, "the whole workload: quantize X and W, fp64 GEMM (NumPy)"


WORKLOADS = {W.name: W for W in (NvfpStudentT, NvfpStudentT46, Nvfp2dWeight, NvfpMseWeight, HadamardMxGemm,
                                  HadamardMxGemm128, FusedMxLinear, VitLinears, LlamaNvfp4, MxLinear128)}


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


def _nv_single_pass(rows, cols, num_sms):
    """Whether the library quantizes an NVFP4 tensor (no caller-given tensor scale, contiguous rows)
    in its single-pass amax+quantize kernel: the dispatch rule of the C library (each SM stages
    ceil(ceil(rows*cols/256) / SMs) 512-byte tiles in at most 227 KB - 2 KB of shared memory)."""
    tiles = (rows * (cols // 8) + 31) // 32
    per = (tiles + num_sms - 1) // num_sms
    return per * 512 <= 227 * 1024 - 2048


def _timed_steps(W, steps, torch, pg):
    """K steps bracketed by a barrier + synchronize on both sides; returns (ms per step, max over
    ranks; host window of the timed region)."""
    _barrier(torch, pg)
    t0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        # bracketed workloads run the steps bare: events between kernels would serialize their
        # launches (no programmatic dependent launch overlap) and add ~3 us each
        W.step(i, timed=not W.bracket)
    end.record()
    torch.cuda.synchronize()
    t1 = time.time()
    _barrier(torch, pg)
    local_ms = start.elapsed_time(end) if W.bracket else W.timed_ms_total()
    return _max_over_ranks(torch, pg, local_ms) / steps, (t0, t1)


def _attribution(W, steps, torch, pg, F):
    """Per-family device time per step.  For bracketed workloads a second pass of the same steps with
    CUDA events around every launch (its per-launch durations include the event-serialized launch
    gaps, so the kernels' rates are conservative against the headline pass)."""
    attr_steps = steps
    if W.bracket:
        attr_steps = max(3, min(steps, 1000))
        _barrier(torch, pg)
        for i in range(attr_steps):
            W.step(i, timed=True)
        torch.cuda.synchronize()
        F.fp4_check_device_errors()
    fam_ms = {k: sum(a.elapsed_time(b) for a, b in tm.pairs) / attr_steps for k, tm in W.timers.items() if tm.pairs}
    return attr_steps, fam_ms


def _solo_times(W, steps, torch, pg):
    """Per-step device time of each kernel family timed alone: its launches back to back (inputs
    rotating past L2 as in the step), bracketed by one CUDA event pair, after warm-up.  Unlike events
    around every launch of the step, this keeps programmatic dependent launch overlapping each
    launch's setup with the previous one's tail, as in the timed step; None if the workload has no
    per-family calls."""
    calls = W.solo_calls() if hasattr(W, "solo_calls") else None
    if not calls:
        return None
    n = max(3, min(steps, 200))
    out = {}
    for key, (fn, launches) in calls.items():
        for i in range(3):
            fn(i)
        _barrier(torch, pg)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(n):
            fn(i)
        b.record()
        torch.cuda.synchronize()
        out[key] = a.elapsed_time(b) / n * launches
    return out


def _roofline(W, fam_ms, attr_steps, torch, pg, device, solo_ms=None):
    """Roofline of the dominant single-kernel family (largest share of device time) and the rates of
    every family.  With solo_ms (per-family times from _solo_times) those set the rates; the
    in-step event times are kept beside them."""
    events_ms = fam_ms
    if solo_ms:
        fam_ms = {k: solo_ms.get(k, v) for k, v in fam_ms.items()}
    dom = max((k for k in fam_ms if k in W.single_kernel()), key=lambda k: fam_ms[k])
    dom_ms = _max_over_ranks(torch, pg, fam_ms[dom])
    peaks = _peaks()
    if W.family_bound(dom) == "tensor":
        # dense FP4 peak = measured bf16 GEMM peak x 4 (nominal FP4 : bf16 ratio, 9 : 2.25 PFLOP/s).
        # The burst figure: the timed runs are short and the clock record shows no power capping;
        # the fraction of the sustained figure is given beside it.
        achieved = W.family_work(dom) / (dom_ms * 1e-3) / 1e12
        peak = 4.0 * peaks["bf16_tflops"]
        roofline = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1),
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": _load_traffic(W.name, dom),
                    "peak_source": peaks["source"] + " (bf16 burst x 4)",
                    "frac_of_sustained_peak": round(achieved / (4.0 * peaks["bf16_tflops_sustained"]), 4)}
    elif W.family_bound(dom) == "alu":
        # instruction-issue bound: work in candidate evaluations, peak = SMs x 4 sub-partitions x 32
        # lanes x max SM clock / instructions per evaluation (see the workload's alu_peak)
        sms = torch.cuda.get_device_properties(device).multi_processor_count
        peak, per_eval = W.alu_peak(sms)
        achieved = W.family_work(dom) / (dom_ms * 1e-3) / 1e9
        roofline = {"kernel": dom, "bound": "alu", "achieved": round(achieved, 1), "peak": round(peak / 1e9, 1),
                    "unit": "Geval/s", "frac": round(achieved * 1e9 / peak, 4), "traffic": _load_traffic(W.name, dom),
                    "peak_source": f"derived: {sms} SMs x 128 lanes x 1965 MHz / {per_eval} instructions per evaluation"}
    else:
        achieved = W.family_work(dom) / (dom_ms * 1e-3) / 1e9
        roofline = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                    "traffic": _load_traffic(W.name, dom), "peak_source": peaks["source"]}
    l2w = _load_counter(W.name, dom, "l2_write_bytes_per_launch")
    if l2w is not None:
        # DRAM writes of a launch miss what is still in L2 when it ends; the bytes the SMs wrote
        # to L2 confirm the written side instead
        rd = _load_counter(W.name, dom, "dram_read_bytes_per_launch")
        roofline["traffic_l2_writes"] = l2w
        if rd is not None:
            alg = W.family_work(dom) / (W.family_launches(dom) if hasattr(W, "family_launches") else 1)
            roofline["traffic_read_plus_l2_writes_over_algorithmic"] = round((rd + l2w) / alg, 4)
    issue = _issue_roofline(W, dom, dom_ms, torch, device)
    if issue is not None:
        roofline["issue"] = issue
    per_family = {}
    for k, ms in fam_ms.items():
        work = W.family_work(k)
        if W.family_bound(k) == "tensor":
            per_family[k] = {"us_per_step": round(ms * 1e3, 2), "tflops": round(work / (ms * 1e-3) / 1e12, 1)}
        elif W.family_bound(k) == "alu":
            per_family[k] = {"us_per_step": round(ms * 1e3, 2), "geval_s": round(work / (ms * 1e-3) / 1e9, 1)}
        else:
            per_family[k] = {"us_per_step": round(ms * 1e3, 2), "gbs": round(work / (ms * 1e-3) / 1e9, 1)}
    if solo_ms:
        for k in per_family:
            per_family[k]["us_per_step_events_in_step"] = round(events_ms[k] * 1e3, 2)
        roofline["timing"] = ("per-kernel times: each family's launches alone, back to back, one CUDA event pair; "
                              "us_per_step_events_in_step: events around every launch of the step")
    roofline["per_kernel"] = per_family
    roofline["attribution_steps"] = attr_steps
    return roofline


def _issue_roofline(W, dom, dom_ms, torch, device):
    """Instruction-issue roofline of the dominant kernel when ncu counted its instructions
    (profiles/traffic.json: warp instructions executed per launch, from the same capture as its DRAM
    bytes): achieved issue rate = counted warp instructions per step / device time; peak = SMs x 4
    sub-partitions x 1 warp instruction per cycle x max SM clock."""
    inst = _load_counter(W.name, dom, "warp_inst_per_launch")
    if inst is None:
        return None
    launches = W.family_launches(dom) if hasattr(W, "family_launches") else 1
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    peak = sms * 4 * 1965e6
    achieved = inst * launches / (dom_ms * 1e-3)
    elems = W.family_elements(dom) if hasattr(W, "family_elements") else None
    out = {"bound": "alu", "achieved": round(achieved / 1e9, 1), "peak": round(peak / 1e9, 1),
           "unit": "G warp instructions/s", "frac": round(achieved / peak, 4),
           "peak_source": f"derived: {sms} SMs x 4 schedulers x 1 warp instruction per cycle x 1965 MHz",
           "warp_inst_per_launch": inst}
    if elems:
        out["thread_inst_per_element"] = round(inst * 32 * launches / elems, 2)
    return out


def _run_companion(args, torch, F, device, pg, sampler):
    """The block-scaled GEMM half of the metric, measured in the same process as the default
    workload: rotate + quantize X[8192, 4096] with b = 128, then the MXFP4 GEMM against the offline
    W[11008, 4096] with bf16 output, timed under the same clock sampler."""
    W = HadamardMxGemm128(torch, F)
    W.setup(device)
    for i in range(max(3, min(args.warmup, 10))):
        W.step(i)
    F.fp4_check_device_errors()
    steps = max(3, min(args.steps, 300))
    ms_step, window = _timed_steps(W, steps, torch, pg)
    F.fp4_check_device_errors()
    attr_steps, fam_ms = _attribution(W, steps, torch, pg, F)
    solo = _solo_times(W, steps, torch, pg)
    F.fp4_check_device_errors()
    roofline = _roofline(W, fam_ms, attr_steps, torch, pg, device, solo)
    out = {"workload": W.name, "metric": "block-scaled FP4 GEMM TFLOP/s (GEMM flops / step time incl. rotate+quantize)",
           "value": round(W.value_from_ms(ms_step, 1), 1), "unit": W.unit, "steps": steps,
           "ms_per_step": round(ms_step, 5), "config": W.config(), "roofline": roofline,
           "gpu_launches": W.launches_per_step * steps, "window": window}
    W.release()
    return out


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
    if isinstance(W, LlamaNvfp4):
        sms = torch.cuda.get_device_properties(device).multi_processor_count
        W.launches_per_step = sum(1 + (1 if _nv_single_pass(m, k, sms) else 2) for k, n, m in W.cases)

    for i in range(args.warmup):
        W.step(i)
    F.fp4_check_device_errors()

    sampler = ClockSampler(_smi_id(torch, local))
    sampler.start()
    time.sleep(0.3)                              # let the sampler produce its first line
    ms_step, window = _timed_steps(W, args.steps, torch, pg)
    sampler.t_start, sampler.t_end = window
    F.fp4_check_device_errors()
    value = W.value_from_ms(ms_step, ws)
    attr_steps, fam_ms = _attribution(W, args.steps, torch, pg, F)
    solo = _solo_times(W, args.steps, torch, pg)
    F.fp4_check_device_errors()
    roofline = _roofline(W, fam_ms, attr_steps, torch, pg, device, solo)
    cases = W.cases_summary(args.steps) if hasattr(W, "cases_summary") else None

    # end to end through the public API with host buffers: pinned H2D of the step's inputs, the
    # step, D2H of every output
    outs = W.outputs()
    host_outs = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
    e2e_steps = max(3, min(20, args.steps))
    for _ in range(2):
        W.e2e_step(host_outs)
    _barrier(torch, pg)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        h2d, d2h = W.e2e_step(host_outs)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(torch, pg, e0.elapsed_time(e1)) / e2e_steps
    e2e = {"value": round(W.value_from_ms(e2e_ms, ws), 2), "unit": W.unit, "ms_per_step": round(e2e_ms, 4),
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    companion = None
    if getattr(W, "gemm_companion", False) and not args.no_gemm:
        companion = _run_companion(args, torch, F, device, pg, sampler)
        time.sleep(0.25)                         # the sampler's last line inside the window
    sampler.stop()
    clocks = sampler.summary()
    if companion is not None:
        companion["clocks"] = sampler.summary(*companion.pop("window"))

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = _cpu_baseline(W)
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
    if cases is not None:
        line["cases"] = cases
    if companion is not None:
        line["gemm"] = companion
    print(json.dumps(line), flush=True)


def _smi_id(torch, local):
    """nvidia-smi -i selector of this process's GPU (its UUID; the index as a fallback)."""
    try:
        u = str(torch.cuda.get_device_properties(local).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(local)


def _sources_hash(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _load_counter(workload, kernel, key):
    """A per-launch ncu figure of `kernel` from the committed captures (profiles/traffic.json), or
    None when none exists or the kernel's sources changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(workload, {}).get(kernel)
    if not d or d.get("sources_sha256_16") != _sources_hash(d.get("sources", [])):
        return None
    return d.get(key)


def _load_traffic(workload, kernel):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu capture."""
    return _load_counter(workload, kernel, "dram_bytes_per_launch")


def _scale_work(W, work, seconds):
    return work / seconds / (1e12 if W.unit == "TFLOP/s" else 1e9)


def _one_thread():
    """Context that holds NumPy's BLAS to one thread, so the oracle's timing uses exactly one core."""
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=1)


def _cpu_baseline(W):
    """The oracle as it stands, on a bounded sample of the workload, on one host core."""
    W.oracle_setup()
    rows, desc = W.cpu_sample()
    with _one_thread():
        t0 = time.time()
        work = W.oracle_step(rows)
        dt = time.time() - t0
    return {"value": round(_scale_work(W, work, dt), 6), "unit": W.unit, "cores": 1, "kind": "oracle",
            "sample": desc, "seconds": round(dt, 2), "host_cpus": os.cpu_count()}


def run_reference(args):
    """The oracle as the reference arm: bounded samples of the same workload on host cores."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    W = WORKLOADS[args.workload](None, None)
    W.oracle_setup()
    rows, desc = W.reference_sample()
    with _one_thread():
        for _ in range(args.warmup):
            W.oracle_step(rows)
        t0 = time.time()
        work = 0.0
        for _ in range(args.steps):
            work += W.oracle_step(rows)
        dt = time.time() - t0
    value = _scale_work(W, work, dt)
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": W.unit, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded NumPy PCG64, bf16)",
        "config": dict(W.config(), parallelism="single"), "impl": "reference",
        "cpu_baseline": {"value": round(value, 6), "unit": W.unit, "kind": "oracle", "cores": 1, "sample": desc},
        "e2e": {"value": round(value, 6), "unit": W.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
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
    ap.add_argument("--no-gemm", action="store_true",
                    help="skip the GEMM measurement that the default workload's line carries")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_fp4(args)


if __name__ == "__main__":
    main()
