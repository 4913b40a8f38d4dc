"""Helpers for the GPU parity tests: host<->device transfers of raw bit patterns."""
import numpy as np
import torch


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns (numpy) -> bf16 CUDA tensor with identical bits."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint8)


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def host_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def mixed_input(rows: int, cols: int, seed: int, fmt: str) -> np.ndarray:
    """Heavy-tailed values with per-row scale changes, a zero block, negative
    zeros and bf16 subnormals, as bf16 bit patterns."""
    from workloads import bf16_bits
    g = np.random.default_rng(seed)
    x = (g.standard_t(3, size=(rows, cols)) * 0.1).astype(np.float32)
    span = 20 if fmt == "mxfp4" else 3
    x *= np.exp2(g.integers(-span, span + 1, size=(rows, 1))).astype(np.float32)
    x[0, :min(cols, 32)] = 0.0
    if rows > 1:
        x[1, :8] = -0.0
    if rows > 2 and fmt == "mxfp4":
        x[2, :32] = np.float32(1e-39)
    return bf16_bits(x)
