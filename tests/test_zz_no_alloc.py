"""fp4_amax_noalloc: the allocation-free amax, checked against fp4_amax.

Some callers cannot call cudaMalloc (their allocator already owns all free
device memory, they cannot afford an allocation's synchronization, or they run
inside an allocator callback), so this entry point keeps its scratch in a fixed
array inside the library.  The tests call it through the C ABI: twice in a row
(the array keeps the first call's contents) against the allocating entry
point's result, in a fresh process before anything else of the library has run,
and with the device's free memory read before and after calls on new shapes
(after the warm-up call, a call takes no device memory).  The file is collected
last so that a failure here cannot hide the result of any other test, and it
passes alone in a fresh process.
"""
import ctypes
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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


def test_amax_noalloc_takes_no_device_memory_after_warm_up():
    from microscaling_fp4_quantization_mxfp4_b200 import _lib
    lib = _lib.load()
    g = torch.Generator(device="cuda").manual_seed(99)
    warm = torch.ones((8, 64), dtype=torch.bfloat16, device="cuda")
    xs = [(torch.randn(s, device="cuda", generator=g) * 2.0).to(torch.bfloat16)
          for s in ((1, 8), (777, 1032), (2048, 8192), (8192, 8192))]
    outs = [torch.full((1,), -1.0, dtype=torch.float32, device="cuda") for _ in xs]
    wout = torch.empty((1,), dtype=torch.float32, device="cuda")
    assert _call_noalloc(lib, warm, wout) == 0            # warm-up: the set-up is done here
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for x, out in zip(xs, outs):
        assert _call_noalloc(lib, x, out) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    for x, out in zip(xs, outs):
        assert out.item() == x.float().abs().max().item()


_FRESH = r"""
import ctypes, sys
import torch
sys.path.insert(0, sys.argv[1])
from microscaling_fp4_quantization_mxfp4_b200 import _lib
lib = _lib.load()
x = (torch.arange(4096 * 520, device="cuda", dtype=torch.float32).reshape(4096, 520) % 977 - 400).to(torch.bfloat16)
want = x.float().abs().max().item()
out = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
st = torch.cuda.current_stream().cuda_stream
for _ in range(2):
    out.fill_(-1.0)
    r = lib.fp4_amax_noalloc(ctypes.c_void_p(x.data_ptr()), 4096, 520, 520, ctypes.c_void_p(out.data_ptr()),
                             ctypes.c_void_p(st))
    assert r == 0, r
    assert out.item() == want, (out.item(), want)
print("fresh ok", want)
"""


def test_amax_noalloc_first_in_a_fresh_process():
    """The entry point's first call in a process, before any other call into the library (so
    before the allocating entry points' scratch exists), gives the exact amax, twice."""
    r = subprocess.run([sys.executable, "-c", _FRESH, ROOT], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "fresh ok" in r.stdout


def test_amax_noalloc_rejects_inputs_beyond_its_scratch():
    from microscaling_fp4_quantization_mxfp4_b200 import _lib
    lib = _lib.load()
    x = torch.empty((8192, 8200), dtype=torch.bfloat16, device="cuda")   # 2^26 + 65536 elements
    out = torch.empty((1,), dtype=torch.float32, device="cuda")
    assert _call_noalloc(lib, x, out) == -2                               # FP4_ERR_SHAPE, nothing launched
