"""bench.py's host-side contract, on CPU: the reference arm (the oracle on a bounded sample)
prints one JSON line with the keys the harness reads, for every workload."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("workload", ["mx_linear_128x512", "nvfp4_student_t_4096", "nvfp4_4o6_student_t_4096",
                                      "nvfp4_2d_weight_11008x4096", "nvfp4_mse_weight_11008x4096",
                                      "mxfp4_fused_linear_8192x11008x4096"])
def test_reference_arm_line(workload):
    d = _run("--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "3")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["config"]["workload"] == workload
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_warmup_floor():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], capture_output=True,
                         text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0


def test_single_pass_rule_matches_library_bound():
    import bench
    # 4096 x 4096 bf16 on 148 SMs: 227 tiles of 512 B per SM = 116,224 B <= 227 KB - 2 KB
    assert bench._nv_single_pass(4096, 4096, 148)
    assert not bench._nv_single_pass(16384, 11008, 148)
    assert bench._nv_single_pass(1, 4096, 148)


def test_reference_arm_two_ranks():
    """Launched as the harness launches N > 1 (torchrun, two ranks on 127.0.0.1): rank 0 alone
    prints the one JSON line, with n_gpus = 2; the other rank exits 0 without output."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "mx_linear_128x512", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
