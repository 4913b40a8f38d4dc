"""Pins for the oracle's Philox4x32-10 (CPU only)."""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest

from oracle.philox import philox4x32_10, philox_words

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_known_answer_vectors():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) if l[0] != "#" and l.strip()]
    assert len(rows) >= 3
    for r in rows:
        v = [int(t, 16) for t in r]
        out = philox4x32_10(np.array(v[:4], np.uint64).reshape(4, 1), (v[4], v[5]))
        assert [int(x) for x in out[:, 0]] == v[6:]


def test_stream_mapping():
    # element idx takes word idx & 3 of the block counter idx >> 2
    seed = (0x12345678 << 32) | 0x9ABCDEF0
    idx = np.arange(64, dtype=np.uint64)
    w = philox_words(seed, idx)
    for j in range(16):
        out = philox4x32_10(np.array([j, 0, 0, 0], np.uint64).reshape(4, 1), (0x9ABCDEF0, 0x12345678))
        np.testing.assert_array_equal(w[4 * j: 4 * j + 4], out[:, 0])
    # high counter word carries idx >> 34
    big = np.array([(1 << 34) + 5], np.uint64)
    out = philox4x32_10(np.array([1, 1, 0, 0], np.uint64).reshape(4, 1), (0x9ABCDEF0, 0x12345678))
    assert philox_words(seed, big)[0] == out[1, 0]


def test_words_look_uniform():
    w = philox_words(1, np.arange(1 << 18, dtype=np.uint64)).astype(np.float64)
    assert abs(w.mean() / 2 ** 32 - 0.5) < 0.005
    hist = np.histogram(w, bins=16, range=(0, 2 ** 32))[0]
    assert hist.min() > 0.9 * hist.mean()


_TRITON_SNIPPET = textwrap.dedent("""
    import os, sys, json
    os.environ["TRITON_INTERPRET"] = "1"
    import torch, triton, triton.language as tl

    @triton.jit
    def k(out_ptr, c0_ptr, c1_ptr, k0, k1, N: tl.constexpr):
        i = tl.arange(0, N)
        c0 = tl.load(c0_ptr + i).to(tl.uint32)
        c1 = tl.load(c1_ptr + i).to(tl.uint32)
        z = tl.zeros([N], dtype=tl.uint32)
        a, b, c, d = tl.philox_impl(c0, c1, z, z, k0.to(tl.uint32), k1.to(tl.uint32), 10)
        tl.store(out_ptr + i * 4 + 0, a)
        tl.store(out_ptr + i * 4 + 1, b)
        tl.store(out_ptr + i * 4 + 2, c)
        tl.store(out_ptr + i * 4 + 3, d)

    N = 256
    c0 = torch.arange(N, dtype=torch.int64) * 977 + 12345
    c1 = torch.arange(N, dtype=torch.int64) % 7
    out = torch.zeros(4 * N, dtype=torch.int32)
    k[(1,)](out, c0.to(torch.int32), c1.to(torch.int32), int(sys.argv[1]), int(sys.argv[2]), N=N)
    print(json.dumps([v & 0xffffffff for v in out.tolist()]))
""")


@pytest.mark.parametrize("key", [(0, 0), (1, 0), (0x9ABCDEF0, 0x12345678)])
def test_matches_triton_interpreter(key, tmp_path):
    """Independent library implementation (Triton's philox, run on the CPU interpreter)."""
    pytest.importorskip("triton")
    script = tmp_path / "tri.py"
    script.write_text(_TRITON_SNIPPET)
    env = dict(os.environ, TRITON_INTERPRET="1", CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, str(script), str(key[0]), str(key[1])], capture_output=True,
                         text=True, env=env, timeout=600)
    if res.returncode != 0:
        pytest.skip("triton interpreter unavailable: " + res.stderr.strip().splitlines()[-1][:200])
    import json
    got = np.array(json.loads(res.stdout.strip().splitlines()[-1]), np.uint64).reshape(-1, 4).T
    N = got.shape[1]
    c0 = np.arange(N, dtype=np.uint64) * 977 + 12345
    c1 = np.arange(N, dtype=np.uint64) % 7
    ctr = np.stack([c0, c1, np.zeros(N, np.uint64), np.zeros(N, np.uint64)])
    np.testing.assert_array_equal(philox4x32_10(ctr, key), got)
