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


MUTANTS = {
    "range rounding": (r"return c \* sp\.q \+ min\(c, sp\.r\);", "return c * sp.q + min(c, sp.r + 1);"),
    "owner of a step": (r"return x < big \? x / \(sp\.q \+ 1\) : sp\.r \+ \(x - big\) / sp\.q;",
                        "return x < big ? x / sp.q : sp.r + (x - big) / sp.q;"),
    "K-block wrap": (r"\} else if \(\+\+kb == KB\) \{", "} else if (++kb == KB + 1) {"),
    "first segment end": (r"first_end = min\(e, \(b / KB \+ 1\) \* KB\);", "first_end = min(e, (b / KB + 1) * KB - 1);"),
    "cluster range end": (r"\*e = t \* KB \+ \(r \+ 1\) \* KB / C;", "*e = t * KB + (r + 1) * (KB / C);"),
}
PREFILL_MUTANTS = {
    "piece offset": (r"off = \(j % p\.split\) \* cols;", "off = 0;"),
    "tile index in group": (r"const int r = t - g \* per_group;", "const int r = t - g * per_group + 1;"),
    "item count": (r"\(tail - 1 - c\) / G \+ 1 : 0\);", "(tail - 1 - c) / G : 0);"),
    "last group's height": (r"const int gm = min\(p\.group_m, p\.num_m - first_m\);", "const int gm = p.group_m;"),
}


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc")
@pytest.mark.parametrize("name", sorted(MUTANTS) + sorted(PREFILL_MUTANTS))
def test_schedule_check_catches_planted_mistake(name):
    """A plausible mistake planted in a copy of the decode or prefill schedule fails the check."""
    import re
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    root = os.path.dirname(HERE)
    pat, rep = MUTANTS[name] if name in MUTANTS else PREFILL_MUTANTS[name]
    header = "sched.cuh" if name in MUTANTS else "gemm_prefill.cuh"
    with tempfile.TemporaryDirectory() as tmp:
        shutil.copytree(os.path.join(root, "fp8_w8a8_quantized_amax_b200", "csrc"),
                        os.path.join(tmp, "fp8_w8a8_quantized_amax_b200", "csrc"))
        os.makedirs(os.path.join(tmp, "tests"))
        shutil.copy(os.path.join(HERE, "schedule_check.cu"), os.path.join(tmp, "tests"))
        hdr = os.path.join(tmp, "fp8_w8a8_quantized_amax_b200", "csrc", header)
        src, n = re.subn(pat, rep, open(hdr).read())
        assert n >= 1, f"mutation '{name}' did not apply"
        open(hdr, "w").write(src)
        exe = os.path.join(tmp, "schedule_check")
        subprocess.check_call([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a", "-x", "cu",
                               os.path.join(tmp, "tests", "schedule_check.cu"), "-o", exe], timeout=300)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "FAIL" in r.stdout, f"planted mistake '{name}' passed the schedule check"
