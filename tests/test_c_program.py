"""The boundary is a C ABI: a plain C99 program (gcc, -pedantic -Werror)
includes include/fp8q.h, links libfp8q.so and calls it.  On a machine without
a GPU it checks the calls that need none: version, status strings, argument
validation before any CUDA call, the empty-input no-ops, and that a valid
call reports FP8Q_ERR_CUDA."""
import os
import shutil
import subprocess
import tempfile

import pytest
import torch

import fp8_w8a8_quantized_amax_b200 as fq
from fp8_w8a8_quantized_amax_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "fp8q.h"

#define CHECK(cond) do { if (!(cond)) { printf("failed: %s (line %d)\n", #cond, __LINE__); return 1; } } while (0)

int main(int argc, char** argv) {
    int no_gpu = argc > 1 && strcmp(argv[1], "no-gpu") == 0;
    void* p = (void*)0x10000;               /* aligned dummy device address, never dereferenced */
    CHECK(fp8q_version() > 0);
    CHECK(strncmp(fp8q_status_string(FP8Q_OK), "FP8Q", 4) == 0);
    CHECK(fp8_quant_act(NULL, 4, 256, 256, FP8Q_CHANNEL_TOKEN, p, 256, p, NULL) == FP8Q_ERR_INVALID_ARG);
    CHECK(fp8_quant_weight(p, 64, 24, 24, FP8Q_CHANNEL_TOKEN, p, 24, p, NULL) == FP8Q_ERR_INVALID_ARG);
    CHECK(fp8_linear(p, p, p, p, 4, 64, 256, 7, p, 64, p, 1 << 20, NULL) == FP8Q_ERR_INVALID_ARG);
    CHECK(fp8_linear(NULL, NULL, NULL, NULL, 0, 64, 256, FP8Q_CHANNEL_TOKEN, NULL, 64, NULL, 0, NULL) == FP8Q_OK);
    CHECK(fp8_linear_w8a16(p, 256, p, p, 65, 64, 256, p, 64, p, 1 << 20, NULL) == FP8Q_ERR_UNSUPPORTED);
    if (no_gpu) {
        CHECK(fp8_quant_act(p, 4, 256, 256, FP8Q_CHANNEL_TOKEN, p, 256, p, NULL) == FP8Q_ERR_CUDA);
        CHECK(fp8_linear_workspace_size(8, 8192, 8192, FP8Q_CHANNEL_TOKEN) == 0);
    }
    printf("ok\n");
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_links_and_calls_the_library():
    fbuild.build()
    libdir = os.path.dirname(fq.LIB_PATH)
    with tempfile.TemporaryDirectory() as tmp:
        src = os.path.join(tmp, "prog.c")
        exe = os.path.join(tmp, "prog")
        open(src, "w").write(PROGRAM)
        subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                               "-I", os.path.join(ROOT, "include"), src, "-o", exe,
                               "-L", libdir, "-l:" + os.path.basename(fq.LIB_PATH), "-Wl,-rpath," + libdir])
        args = [exe] + ([] if torch.cuda.is_available() else ["no-gpu"])
        r = subprocess.run(args, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
