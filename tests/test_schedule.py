"""The decode kernel's stream-K schedule, checked on the host: the kernel's own
step iterator and range functions are compiled by nvcc for the CPU and run
over every small (tiles, K blocks, CTAs) case and the Llama decode shapes
(tests/schedule_check.cu lists the invariants).  No GPU is used."""
import os
import shutil
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc")
def test_stream_k_schedule_invariants():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "schedule_check")
        subprocess.check_call([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a", "-x", "cu",
                               os.path.join(HERE, "schedule_check.cu"), "-o", exe], timeout=300)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:]
    assert r.stdout.strip().splitlines()[-1].startswith("ok:")
