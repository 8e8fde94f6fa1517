"""GPU weight-only FP8 linear (bf16 activations, E4M3 weights dequantized in
the kernel: the CUDA-core kernel for one token, the tensor-core decode schedule
with widened weight tiles for 2..64) vs the oracle.

The weights are quantized by the oracle (the codes are shown bit-exact with
the GPU quantizer elsewhere); both sides take the same codes, scales and bf16
activations, and the outputs must agree within 4e-3 * max|y_ref| + 1 bf16 ulp
elementwise.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import synth
import fp8_w8a8_quantized_amax_b200 as fq
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from fp8_w8a8_quantized_amax_b200 import build
    build.build()
    fq.device_error(clear=True)
    yield
    assert fq.device_error(clear=True) == 0


def check(M, N, K, seed=0, ldx_pad=0, ldy_pad=0, rows=None):
    x = synth.make_x(M, K, seed=seed)
    w = synth.make_w(N, K, seed=seed)
    wq, ws = oracle.quant_rows(w)
    xd = x.to(DEV)
    if ldx_pad:
        xfull = torch.zeros((M, K + ldx_pad), dtype=torch.bfloat16, device=DEV)
        xfull[:, :K] = xd
        xd = xfull[:, :K]
    out = None
    if ldy_pad:
        yfull = torch.full((M, N + ldy_pad), 7.0, dtype=torch.bfloat16, device=DEV)
        out = yfull[:, :N]
    y = fq.fp8_linear_w8a16(xd, torch.from_numpy(wq).to(DEV), torch.from_numpy(ws).to(DEV), out=out)
    torch.cuda.synchronize()
    if ldy_pad:
        assert torch.all(yfull[:, N:] == 7.0), "columns past N were written"
    y = y.float().cpu().numpy()
    if rows is None:
        P.assert_y_close(y, oracle.linear_w8a16(x, wq, ws), what=f"W8A16 {M}x{N}x{K}")
    else:
        # rows of the weight are independent: the oracle computes only the sampled channels
        ref = oracle.linear_w8a16(x, np.ascontiguousarray(wq[rows]), np.ascontiguousarray(ws[rows]))
        P.assert_y_close(y[:, rows], ref, what=f"W8A16 {M}x{N}x{K} sampled")


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 11, 16, 17, 31, 32, 33, 48, 64])
def test_w8a16_every_token_count(M):
    # K = 4096 + 16: a ragged last K block (and, for one token, a whole stage
    # then one 16-code lane); N = 1001: a ragged last weight tile / CTA
    check(M, 1001, 4112, seed=M)


@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (2, 7, 32), (16, 3, 512), (4, 128, 12288), (8, 513, 8192),
                                   (64, 130, 144), (40, 4096, 256)])
def test_w8a16_small_and_odd_shapes(M, N, K):
    check(M, N, K, seed=N)


def test_w8a16_strided_activations_and_output():
    check(5, 300, 2048, seed=9, ldx_pad=40, ldy_pad=12)


@pytest.mark.parametrize("M,N,K", [(1, 57344, 8192), (8, 8192, 28672), (16, 10240, 8192), (64, 57344, 8192)])
def test_w8a16_llama70b_shapes_sampled(M, N, K):
    # full Llama-3.1-70B decode shapes (gate+up, down, qkv); oracle on 96 sampled channels
    rng = np.random.default_rng(N + M)
    rows = np.unique(np.concatenate([rng.choice(N, 94, replace=False), [0, N - 1]]))
    check(M, N, K, seed=M, rows=rows)


def test_w8a16_every_code_widens_exactly():
    # one-hot activations pick one code per channel: Y[m, n] = bf16(E4M3(n)), no
    # rounding anywhere, so any inexact widening (a flushed subnormal, a lost
    # sign) shows; all 254 finite codes, both kernels.  Values are compared
    # (-0 == +0): the sum for the -0 code starts from +0, as the oracle's does.
    K = 256
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    N = codes.size
    wq = np.zeros((N, K), np.uint8)
    wq[:, 37] = codes
    ws = np.ones(N, np.float32)
    vals = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float()
    for M in (1, 2, 16):
        x = torch.zeros(M, K, dtype=torch.bfloat16)
        x[:, 37] = 1.0
        y = fq.fp8_linear_w8a16(x.to(DEV), torch.from_numpy(wq).to(DEV), torch.from_numpy(ws).to(DEV))
        want = vals.to(torch.bfloat16).expand(M, N)
        assert torch.equal(y.cpu().float(), want.float()), f"M={M}"


def test_w8a16_zero_activations_and_codes():
    K, N = 1024, 64
    wq = np.zeros((N, K), np.uint8)
    wq[:, ::2] = 0x80                       # -0.0 codes
    ws = np.full(N, 0.5, np.float32)
    x = synth.make_x(3, K, seed=1).to(DEV)
    y = fq.fp8_linear_w8a16(x, torch.from_numpy(wq).to(DEV), torch.from_numpy(ws).to(DEV))
    assert torch.all(y == 0)
    w = synth.make_w(N, K, seed=2)
    wq, ws = oracle.quant_rows(w)
    y = fq.fp8_linear_w8a16(torch.zeros(3, K, dtype=torch.bfloat16, device=DEV), torch.from_numpy(wq).to(DEV),
                            torch.from_numpy(ws).to(DEV))
    assert torch.all(y == 0)


def test_w8a16_matches_w8a8_layer_loosely():
    # the same weights with quantized activations differ only by the activation rounding
    M, N, K = 4, 512, 4096
    x = synth.make_x(M, K, seed=5).to(DEV)
    w = synth.make_w(N, K, seed=5).to(DEV)
    wq, ws = fq.fp8_quant_weight(w)
    y16 = fq.fp8_linear_w8a16(x, wq, ws).float()
    xq, xs = fq.fp8_quant_act(x)
    y8 = fq.fp8_linear(xq, xs, wq, ws).float()
    assert (y16 - y8).abs().max() <= 0.1 * y16.abs().max()


@pytest.mark.parametrize("kernel,M,N,K", [("cuda", 2, 1001, 4112), ("cuda", 8, 520, 8192), ("cuda", 16, 300, 4096),
                                          ("tc", 1, 1001, 4112), ("widen8", 2, 1001, 4112), ("widen8", 17, 520, 8192),
                                          ("widen8", 64, 300, 4096), ("exact-cuda", 2, 0, 0), ("exact-tc", 1, 0, 0)])
def test_w8a16_forced_kernel(kernel, M, N, K):
    # both kernels on token counts the default dispatch gives to the other one,
    # and the tensor-core kernel with eight widen warps instead of four
    # ("exact-*": the every-code test under that choice)
    env = dict(os.environ)
    if kernel == "widen8":
        env["FP8Q_W16_WIDEN"] = "8"
    else:
        env["FP8Q_W8A16_KERNEL"] = kernel.replace("exact-", "")
    if kernel.startswith("exact-"):
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                            __file__ + "::test_w8a16_every_code_widens_exactly"],
                           env=env, capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
        return
    r = subprocess.run([sys.executable, "-m", "tests._forced_kernel", "w8a16", str(M), str(N), str(K)],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


def test_w8a16_workspace_reuse_leaves_it_zero():
    shapes = [(8, 8192, 8192), (3, 1001, 4112), (64, 4096, 1024), (2, 57344, 256)]
    need = max(fq.fp8_linear_w8a16_workspace_size(*s_) for s_ in shapes)
    wk = torch.zeros(need, dtype=torch.uint8, device=DEV)
    for i, (M, N, K) in enumerate(shapes):
        x = synth.make_x(M, K, seed=i)
        w = synth.make_w(N, K, seed=i)
        wq, ws = oracle.quant_rows(w)
        rows = np.arange(0, N, max(1, N // 64))
        y = fq.fp8_linear_w8a16(x.to(DEV), torch.from_numpy(wq).to(DEV), torch.from_numpy(ws).to(DEV), workspace=wk)
        torch.cuda.synchronize()
        assert int(wk.count_nonzero()) == 0
        ref = oracle.linear_w8a16(x, np.ascontiguousarray(wq[rows]), np.ascontiguousarray(ws[rows]))
        P.assert_y_close(y.float().cpu().numpy()[:, rows], ref, what=f"W8A16 reuse {M}x{N}x{K}")


def test_w8a16_rejects_more_than_64_tokens():
    x = torch.zeros(65, 256, dtype=torch.bfloat16, device=DEV)
    wq = torch.zeros(32, 256, dtype=torch.uint8, device=DEV)
    ws = torch.ones(32, dtype=torch.float32, device=DEV)
    with pytest.raises(RuntimeError):
        fq.fp8_linear_w8a16(x, wq, ws)
