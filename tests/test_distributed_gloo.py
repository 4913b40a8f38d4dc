"""World-size-2 gloo tests (CPU) of the multi-rank host logic: the NVFP4 tensor-scale exchange for a
row-sharded tensor, the shards' stochastic rounding under their first rows, and the bench's
max-over-ranks timing reduction.  The CUDA amax / tensor-scale / quantize kernels are replaced by
CPU stand-ins here; their parity is tested on the GPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from workloads import bf16_to_f32, nvfp4_student_t


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from microscaling_fp4_quantization_mxfp4_b200.distributed import (shard_rows, sharded_nvfp4_quantize,
                                                                           sharded_nvfp4_tensor_scale)
        import bench
        bits = nvfp4_student_t(256, 512, seed=1)
        x = bf16_to_f32(bits)
        a, b = shard_rows(x.shape[0], world, rank, align=16)
        shard = torch.from_numpy(x[a:b].copy())
        amax_cpu = lambda t: t.abs().max().reshape(1).to(torch.float32)
        scale_cpu = lambda amax: torch.tensor([O.nv_tensor_scale(amax.numpy())], dtype=torch.float32)
        ts = sharded_nvfp4_tensor_scale(shard, amax_fn=amax_cpu, scale_fn=scale_cpu)
        t_max = bench._max_over_ranks(torch, dist, float(rank + 1) * 1.5)

        def quantize_cpu(xs, fmt, rnd, seed, tensor_scale_in, sf_layout, first_row):
            assert sf_layout == "rowmajor"
            return O.quantize_values(xs.numpy(), fmt=fmt, rnd=rnd, seed=seed,
                                     tensor_scale=float(tensor_scale_in.item()), idx_base=first_row * xs.shape[1])

        qs = sharded_nvfp4_quantize(shard, a, rnd="sr", seed=11, amax_fn=amax_cpu, scale_fn=scale_cpu,
                                    quantize_fn=quantize_cpu)
        out[rank] = (a, b, float(ts.item()), t_max, qs["codes"], qs["scales"])
    finally:
        dist.destroy_process_group()


def test_sharded_tensor_scale_quantize_and_timing_reduction():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    x = bf16_to_f32(nvfp4_student_t(256, 512, seed=1))
    full = O.nv_tensor_scale(x)
    ranges = sorted((out[r][0], out[r][1]) for r in range(world))
    assert ranges == [(0, 128), (128, 256)]
    for r in range(world):
        assert out[r][2] == float(full)             # every rank sees the global tensor scale
        assert out[r][3] == 3.0                      # max over ranks of (rank + 1) * 1.5
    # stochastic rounding of the shards, each with its first row passed on, is the whole tensor's
    whole = O.quantize_values(x, fmt="nvfp4", rnd="sr", seed=11)
    parts = sorted(out[r][:1] + out[r][4:] for r in range(world))
    np.testing.assert_array_equal(np.concatenate([p[1] for p in parts]), whole["codes"])
    np.testing.assert_array_equal(np.concatenate([p[2] for p in parts]), whole["scales"])


def test_shard_rows_cover_exactly():
    from microscaling_fp4_quantization_mxfp4_b200.distributed import shard_rows
    for total, world, align in [(4096, 8, 16), (100, 3, 16), (17, 4, 1), (1, 2, 16)]:
        got = [shard_rows(total, world, r, align) for r in range(world)]
        assert got[0][0] == 0 and got[-1][1] == total
        for (a0, b0), (a1, b1) in zip(got, got[1:]):
            assert b0 == a1
        assert all(a % align == 0 for a, _ in got if a < total)
