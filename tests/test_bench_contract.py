"""bench.py's output contract, checked on the CPU: the reference arm (the CPU
oracle) prints one JSON line with the keys the benchmark line carries, and
the GPU arm refuses to run without a GPU instead of falling back."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=300):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_json_line():
    import time
    t0 = time.perf_counter()
    r = run_bench("--impl", "reference", "--workload", "tiny_16x256x512", "--steps", "3", "--warmup", "3")
    wall = time.perf_counter() - t0
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("tiny_16x256x512")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # the timed steps are measured ones: they fit inside the process's own run
    assert d["ms_per_step"] * d["steps"] / 1e3 <= wall
    # the same workload description the GPU arm prints
    sys.path.insert(0, ROOT)
    import bench
    import synth
    assert d["config"] == bench.config_of(synth.workloads()["tiny_16x256x512"], 1, 256)


@pytest.mark.skipif(torch.cuda.is_available(), reason="needs a machine without a CUDA device")
def test_gpu_arm_fails_loudly_without_a_gpu():
    r = run_bench("--workload", "tiny_16x256x512", "--steps", "3", "--warmup", "3")
    assert r.returncode != 0
    assert not any(l.strip().startswith("{") for l in r.stdout.splitlines())


def _free_port():
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        return s_.getsockname()[1]


def test_reference_arm_under_torchrun_prints_once_from_rank_0():
    # the launch the scaling run uses: two ranks; rank 0 alone runs and prints
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
                        os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny_16x256x512",
                        "--gpus", "2", "--steps", "3", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2


def test_launch_count_rule_follows_the_decode_dispatch():
    # the fallback count of the bench's gpu_launches (used where the step graph
    # cannot be inspected): the FP8-Block decode shapes of Llama-3.2-3B take
    # cluster split-K (one kernel); a few-tile block problem, and channel mode
    # with 64 tokens on few steps per CTA, add the reduction kernel
    sys.path.insert(0, ROOT)
    import bench
    import synth
    G = lambda M, N, K, mode: synth.Gemm(name="g", M=M, N=N, K=K, mode=mode, x="x", w="w")
    for M in (1, 16):
        for N, K in ((8192, 3072), (5120, 3072), (3072, 8192)):
            assert bench.launches_of(G(M, N, K, synth.BLOCK128), 148) == 1, (M, N, K)
    assert bench.launches_of(G(16, 1024, 2048, synth.BLOCK128), 148) == 2
    assert bench.launches_of(G(8, 28672, 8192, synth.CHANNEL_TOKEN), 148) == 1
    assert bench.launches_of(G(64, 1024, 1024, synth.CHANNEL_TOKEN), 148) == 2
    assert bench.launches_of(G(512, 28672, 8192, synth.CHANNEL_TOKEN), 148) == 1
