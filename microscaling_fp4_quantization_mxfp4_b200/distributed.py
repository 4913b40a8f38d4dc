"""Multi-rank helpers (one process per GPU, torch.distributed over NCCL).

The quantizer is data-parallel: tensors, row blocks and GEMM tiles are
independent, so N GPUs normally run N independent problems with no
collective.  The one exchange the method has is NVFP4's per-tensor scale when
a single tensor is split by rows across ranks ("FP4 All the Way", Abstract:
NVFP4's E4M3 block scales sit under one tensor scale): every rank needs the
global amax.  That is one max all-reduce of a single fp32 between the local
amax pass and the tensor-scale step; each rank then quantizes its rows with
the shared scale (RTN results equal the unsharded tensor's rows exactly).
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist

from .binding import fp4_amax, fp4_nv_tensor_scale, fp4_quantize


def shard_rows(total_rows: int, world: int, rank: int, align: int = 1) -> Tuple[int, int]:
    """Contiguous row range [start, stop) of `rank`, in multiples of `align` rows."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    units = -(-total_rows // align)
    per = -(-units // world)
    start = min(total_rows, rank * per * align)
    stop = min(total_rows, (rank + 1) * per * align)
    return start, stop


def sharded_nvfp4_tensor_scale(x_shard: torch.Tensor, group=None, *,
                               amax_fn: Optional[Callable] = None,
                               scale_fn: Optional[Callable] = None) -> torch.Tensor:
    """NVFP4 tensor scale of a tensor whose rows are split across the ranks of `group`.

    Local amax (a device fp32 [1]), one all-reduce(MAX) of those 4 bytes, then
    s_t = amax / 2688 on the device.  `amax_fn` / `scale_fn` default to the CUDA
    entry points; they are parameters only so the exchange can be exercised
    without a GPU.
    """
    amax = (amax_fn or fp4_amax)(x_shard)
    dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return (scale_fn or fp4_nv_tensor_scale)(amax)


def sharded_nvfp4_quantize(x_shard: torch.Tensor, first_row: int, group=None, rnd="rtn", seed: int = 0,
                           sf_layout="rowmajor", *, amax_fn: Optional[Callable] = None,
                           scale_fn: Optional[Callable] = None, quantize_fn: Optional[Callable] = None, **kw):
    """NVFP4 quantization of this rank's rows [first_row, first_row + rows) under the global tensor
    scale.  Stochastic rounding draws the Philox words of the whole tensor's element indices
    (fp4_quantize_shard), so the ranks' codes concatenate to the unsharded tensor's, for either
    rounding.  The *_fn parameters default to the CUDA entry points; they exist only so the host
    logic can be exercised without a GPU."""
    ts = sharded_nvfp4_tensor_scale(x_shard, group, amax_fn=amax_fn, scale_fn=scale_fn)
    return (quantize_fn or fp4_quantize)(x_shard, fmt="nvfp4", rnd=rnd, seed=seed, tensor_scale_in=ts,
                                         sf_layout=sf_layout, first_row=first_row, **kw)
