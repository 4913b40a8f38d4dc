"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This module only draws random numbers and rounds them to bf16; it holds none of
the quantization arithmetic.  Every tensor is generated on the host with NumPy's
PCG64 (`default_rng([config_seed, tensor_id])`) in fp32 and rounded to bf16
(round-to-nearest-even, via ml_dtypes).  Arrays are returned as bf16 bit
patterns (uint16) so both sides start from identical bits.

Workloads (shapes and distributions follow the five synthetic configurations of
the hot path; the pages name no dataset, so nothing stands in for one):

* ``mx_linear_128x512``: X[128,512] ~ N(0,1), W[512,512] ~ N(0, 0.02), seed 0.
* ``nvfp4_student_t_4096``: A[4096,4096] = 0.1 * Student-t(nu=3), seed 1.
* ``hadamard_mxfp4_8192x11008x4096``: X[8192,4096] ~ N(0,1) with round(1% of
  4096) = 41 channels (columns) scaled x50; W[11008,4096] ~ N(0, 0.02); seed 2.
* ``vit_b16_linears``: M = 256*197 = 50432 tokens; qkv 768->2304, fc1 768->3072,
  fc2 3072->768; X ~ N(0,1), W ~ N(0,0.02), dY ~ N(0, 1e-3); seed 3.
* ``llama7b_nvfp4``: (K,N) in {(4096,4096),(4096,11008),(11008,4096)};
  X ~ N(0,1) at M=16384 with round(0.5% of K) channels x20; W ~ N(0,0.02);
  seed 4.  Smaller M uses the first M rows.

"N(0, s)" is read as standard deviation s.
"""
from __future__ import annotations

import numpy as np
import ml_dtypes

__all__ = [
    "bf16_bits", "bf16_to_f32", "normal_bf16", "student_t_bf16", "outlier_channels",
    "mx_linear_128x512", "nvfp4_student_t", "hadamard_acts", "hadamard_weights",
    "vit_layer", "llama_acts", "llama_weights", "VIT_LAYERS", "LLAMA_SHAPES", "LLAMA_MS",
    "rng",
]

VIT_TOKENS = 256 * 197
VIT_LAYERS = {"qkv": (768, 2304), "fc1": (768, 3072), "fc2": (3072, 768)}   # name -> (K, N)
LLAMA_SHAPES = [(4096, 4096), (4096, 11008), (11008, 4096)]                 # (K, N)
LLAMA_MS = [1, 16, 128, 1024, 4096, 16384]


def rng(config_seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng([config_seed, tensor_id])


def bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (RNE) and return the raw uint16 bit patterns."""
    return np.ascontiguousarray(x32.astype(np.float32).astype(ml_dtypes.bfloat16)).view(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def normal_bf16(shape, std: float, config_seed: int, tensor_id: int) -> np.ndarray:
    g = rng(config_seed, tensor_id)
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return bf16_bits(x)


def student_t_bf16(shape, nu: float, mult: float, config_seed: int, tensor_id: int) -> np.ndarray:
    g = rng(config_seed, tensor_id)
    x = (g.standard_t(nu, size=shape) * mult).astype(np.float32)
    return bf16_bits(x)


def outlier_channels(k: int, frac: float, config_seed: int, tensor_id: int) -> np.ndarray:
    """Indices of round(frac*k) distinct channels, drawn without replacement."""
    n = int(round(frac * k))
    return np.sort(rng(config_seed, tensor_id).choice(k, n, replace=False))


def _scale_columns(bits: np.ndarray, cols: np.ndarray, factor: float) -> np.ndarray:
    x = bf16_to_f32(bits)
    x[:, cols] *= np.float32(factor)
    return bf16_bits(x)


# --- per-workload generators -------------------------------------------------

def mx_linear_128x512(seed: int = 0):
    """X[128,512] ~ N(0,1), W[512,512] ~ N(0,0.02)."""
    return normal_bf16((128, 512), 1.0, seed, 0), normal_bf16((512, 512), 0.02, seed, 1)


def nvfp4_student_t(rows: int = 4096, cols: int = 4096, seed: int = 1):
    """0.1 * Student-t(nu=3), the heavy-tailed tensor of the NVFP4 quantize/dequantize case."""
    return student_t_bf16((rows, cols), 3.0, 0.1, seed, 0)


def hadamard_acts(m: int = 8192, k: int = 4096, seed: int = 2):
    """X[m,k] ~ N(0,1) with 1% of the k channels scaled x50."""
    x = normal_bf16((m, k), 1.0, seed, 0)
    return _scale_columns(x, outlier_channels(k, 0.01, seed, 2), 50.0)


def hadamard_weights(n: int = 11008, k: int = 4096, seed: int = 2):
    return normal_bf16((n, k), 0.02, seed, 1)


def vit_layer(name: str, m: int = VIT_TOKENS, seed: int = 3):
    """(X[m,K], W[N,K], dY[m,N]) for one ViT-B/16 linear."""
    k, n = VIT_LAYERS[name]
    lid = list(VIT_LAYERS).index(name)
    x = normal_bf16((m, k), 1.0, seed, 10 * lid + 0)
    w = normal_bf16((n, k), 0.02, seed, 10 * lid + 1)
    dy = normal_bf16((m, n), 1e-3, seed, 10 * lid + 2)
    return x, w, dy


def llama_acts(k: int, m: int = 16384, seed: int = 4):
    """X[m,k] ~ N(0,1) with 0.5% of channels x20 (generated at 16384 rows; first m rows used)."""
    x = normal_bf16((16384, k), 1.0, seed, 100 + k)
    x = _scale_columns(x, outlier_channels(k, 0.005, seed, 200 + k), 20.0)
    return np.ascontiguousarray(x[:m])


def llama_weights(k: int, n: int, seed: int = 4):
    return normal_bf16((n, k), 0.02, seed, 300 + k + n)
