"""Pins of the oracle's weight-only FP8 linear (bf16 activations, FP8 weights
dequantized when the layer runs: the A100 path of the Llama-3.1-70B-FP8
explainer, hardware section and FAQ Q1)."""
from fractions import Fraction

import numpy as np
import torch

import oracle
import synth
from tests import _pins


def test_w8a16_exact_on_tiny_cases():
    vals = _pins.e4m3_values_torch()
    rng = np.random.default_rng(3)
    M, N, K = 3, 5, 48
    x = (torch.randn(M, K, generator=torch.Generator().manual_seed(3)) * 4).to(torch.bfloat16)
    wq = rng.integers(0, 256, (N, K)).astype(np.uint8)
    wq[(wq & 0x7F) == 0x7F] = 0x38
    ws = rng.uniform(0.01, 0.2, N).astype(np.float32)
    y = oracle.linear_w8a16(x, wq, ws)
    xf = x.float().numpy()
    for m in range(M):
        for n in range(N):
            e = sum(Fraction(float(xf[m, k])) * Fraction(float(vals[wq[n, k]])) for k in range(K))
            e = float(e * Fraction(float(ws[n])))
            assert abs(float(y[m, n]) - e) <= _pins.f32_ulp(e)


def test_w8a16_equals_float64_matmul_of_dequantized_weights():
    x = synth.make_x(4, 1024, seed=4)
    w = synth.make_w(96, 1024, seed=4)
    wq, ws = oracle.quant_rows(w)
    dec = _pins.e4m3_values_torch()[wq.astype(np.int64)]
    ref = (x.double().numpy() @ dec.T) * ws[None, :].astype(np.float64)
    y = oracle.linear_w8a16(x, wq, ws)
    assert np.allclose(y, ref, rtol=1e-6, atol=1e-30)


def test_w8a16_is_close_to_the_bf16_layer():
    # weight-only quantization: close to the unquantized bf16 layer
    x = synth.make_x(2, 2048, seed=5)
    w = synth.make_w(64, 2048, seed=5)
    wq, ws = oracle.quant_rows(w)
    y = oracle.linear_w8a16(x, wq, ws)
    ref = x.double().numpy() @ w.double().numpy().T
    assert np.abs(y - ref).max() <= 0.05 * np.abs(ref).max()
