"""fp4_amax_noalloc: the allocation-free amax, checked against fp4_amax.

Some callers cannot call cudaMalloc (their allocator already owns all free
device memory, they cannot afford an allocation's synchronization, or they run
inside an allocator callback), so this entry point keeps its scratch in a fixed
array inside the library.  The test calls it twice in a row through the C ABI
(the array keeps the first call's contents) and compares each result with the
allocating entry point's.  It is collected last so that a failure here cannot
hide the result of any other test, and it passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, x, out):
    return lib.fp4_amax_noalloc(ctypes.c_void_p(x.data_ptr()), x.shape[0], x.shape[1], x.stride(0),
                                ctypes.c_void_p(out.data_ptr()),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_amax_noalloc_matches_fp4_amax_on_two_calls():
    import microscaling_fp4_quantization_mxfp4_b200 as F
    from microscaling_fp4_quantization_mxfp4_b200 import _lib
    lib = _lib.load()
    g = torch.Generator(device="cuda").manual_seed(1234)
    # first call: a large tensor (many CTAs); second: a smaller one with a smaller max, so a stale
    # partial or counter left by the first call would show up in the second result
    x1 = (torch.randn((4096, 4096), device="cuda", generator=g) * 3.0).to(torch.bfloat16)
    x2 = (torch.randn((300, 2048), device="cuda", generator=g) * 0.01).to(torch.bfloat16)
    for x in (x1, x2):
        out = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        st = _call_noalloc(lib, x, out)
        assert st == 0, lib.fp4_status_string(st).decode()
        ref = F.fp4_amax(x)
        torch.cuda.synchronize()
        # amax is exact (a max of bf16 magnitudes): the two entry points agree bit for bit
        assert out.item() == ref.item()
        assert out.item() == x.float().abs().max().item()


def test_amax_noalloc_rejects_inputs_beyond_its_scratch():
    from microscaling_fp4_quantization_mxfp4_b200 import _lib
    lib = _lib.load()
    x = torch.empty((8192, 8200), dtype=torch.bfloat16, device="cuda")   # 2^26 + 65536 elements
    out = torch.empty((1,), dtype=torch.float32, device="cuda")
    assert _call_noalloc(lib, x, out) == -2                               # FP4_ERR_SHAPE, nothing launched
