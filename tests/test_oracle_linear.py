"""Pins of the oracle's layer output against exact rational arithmetic,
numpy's float64 matmul (exact here: every product is a multiple of 2^-18 and
every partial sum stays far below 2^53 * 2^-18), and special cases.

The output is the FP8 product with x_scale[m] * w_scale[n] applied
(Llama-3.1-8B-Instruct-FP8-Dynamic explainer, FP8 动态量化 table), or, in
block mode, with x_scale[m, kb] * w_scale[n/128, kb] per 128-wide K slice
(Llama-3.2-3B-Instruct-FP8-Block explainer, quantization_config table).
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _pins

VALS = _pins.e4m3_values_torch()


def _rand_codes(rng, shape):
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38   # no NaN codes
    return c


@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (3, 5, 32), (8, 7, 128), (2, 8, 256), (5, 3, 16)])
def test_channel_equals_exact_rationals(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    xq, wq = _rand_codes(rng, (M, K)), _rand_codes(rng, (N, K))
    xs = rng.uniform(0.001, 3, M).astype(np.float32)
    ws = rng.uniform(0.0001, 0.1, N).astype(np.float32)
    y = oracle.linear(xq, xs, wq, ws, oracle.CHANNEL_TOKEN)
    ex = _pins.exact_linear_channel(xq.tolist(), xs, wq.tolist(), ws)
    for m, n in itertools.product(range(M), range(N)):
        e = float(ex[m][n])
        assert abs(float(y[m, n]) - e) <= 0.5 * _pins.f32_ulp(e) * 1.0000001 + 1e-300, (m, n)


@pytest.mark.parametrize("M,N,K", [(2, 130, 256), (3, 4, 384)])
def test_block_equals_exact_rationals(M, N, K):
    rng = np.random.default_rng(M + N + K)
    xq, wq = _rand_codes(rng, (M, K)), _rand_codes(rng, (N, K))
    xs = rng.uniform(0.001, 3, (M, K // 128)).astype(np.float32)
    ws = rng.uniform(0.0001, 0.1, ((N + 127) // 128, K // 128)).astype(np.float32)
    ns = list(range(N)) if N < 10 else [0, 1, 127, 128, 129]
    y = oracle.linear(xq, xs, wq, ws, oracle.BLOCK128)
    for m in range(M):
        for n in ns:
            e = _pins.exact_linear_block(xq[m:m + 1].tolist(), xs[m:m + 1], wq[n:n + 1].tolist(),
                                         ws[n // 128:n // 128 + 1])[0][0]
            tol = _pins.f32_ulp(float(e)) + 1e-12 * float(np.abs(VALS[xq[m]] * VALS[wq[n]]).sum())
            assert abs(float(y[m, n]) - float(e)) <= tol, (m, n)


def test_channel_matches_numpy_float64_matmul_nonsquare():
    rng = np.random.default_rng(5)
    M, N, K = 13, 29, 512
    xq, wq = _rand_codes(rng, (M, K)), _rand_codes(rng, (N, K))
    xs = rng.uniform(0.01, 1, M).astype(np.float32)
    ws = rng.uniform(0.01, 1, N).astype(np.float32)
    P = VALS[xq] @ VALS[wq].T                       # exact in float64
    ref = ((xs.astype(np.float64)[:, None] * ws.astype(np.float64)[None, :]) * P).astype(np.float32)
    y = oracle.linear(xq, xs, wq, ws, oracle.CHANNEL_TOKEN)
    assert np.array_equal(y, ref)


def test_one_hot_weights_reproduce_dequantized_activations():
    rng = np.random.default_rng(6)
    M, K = 6, 64
    xq = _rand_codes(rng, (M, K))
    xs = rng.uniform(0.01, 1, M).astype(np.float32)
    cols = rng.permutation(K)[:10]
    wq = np.zeros((10, K), np.uint8)
    wq[np.arange(10), cols] = 0x38            # E4M3 1.0
    ws = np.ones(10, np.float32)
    y = oracle.linear(xq, xs, wq, ws, oracle.CHANNEL_TOKEN)
    ref = (VALS[xq[:, cols]] * xs[:, None].astype(np.float64)).astype(np.float32)
    assert np.array_equal(y, ref)


def test_zero_activations_give_zero_output():
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    w = synth.make_w(32, 256)
    xq, xs = oracle.quant_rows(x)
    wq, ws = oracle.quant_rows(w)
    assert np.all(oracle.linear(xq, xs, wq, ws, 0) == 0)


def test_block_with_uniform_scales_reduces_to_channel():
    rng = np.random.default_rng(7)
    M, N, K = 4, 256, 384
    xq, wq = _rand_codes(rng, (M, K)), _rand_codes(rng, (N, K))
    a = rng.uniform(0.1, 1, M).astype(np.float32)
    b = np.array([0.25, 0.5], np.float32)      # one value per 128-row tile
    yb = oracle.linear(xq, np.repeat(a[:, None], 3, 1), wq, np.repeat(b[:, None], 3, 1), 1)
    yc = oracle.linear(xq, a, wq, np.repeat(b, 128), 0)
    np.testing.assert_allclose(yb, yc, rtol=2e-7, atol=0)


def test_common_permutation_of_k_leaves_channel_output_unchanged():
    rng = np.random.default_rng(8)
    M, N, K = 5, 9, 256
    xq, wq = _rand_codes(rng, (M, K)), _rand_codes(rng, (N, K))
    xs, ws = rng.uniform(0.1, 1, M).astype(np.float32), rng.uniform(0.1, 1, N).astype(np.float32)
    p = rng.permutation(K)
    y1 = oracle.linear(xq, xs, wq, ws, 0)
    y2 = oracle.linear(xq[:, p], xs, wq[:, p], ws, 0)
    assert np.array_equal(y1, y2)


def test_linear_at_matches_full_output():
    x = synth.make_x(16, 256, seed=0, n_out=2)
    w = synth.make_w(512, 256, seed=0)
    for mode in (0, 1):
        xq, xs = oracle.quant_act(x, mode)
        wq, ws = oracle.quant_weight(w, mode)
        y = oracle.linear(xq, xs, wq, ws, mode)
        ms = np.array([0, 15, 7, 3]); ns = np.array([0, 511, 128, 300])
        assert np.array_equal(oracle.linear_at(xq, xs, wq, ws, mode, ms, ns), y[ms, ns])


def test_tiny_workload_output_close_to_bf16_matmul():
    # a sanity bound, not a pin: the FP8 layer approximates the bf16 layer
    x = synth.make_x(16, 256, seed=0, n_out=2)
    w = synth.make_w(512, 256, seed=0)
    xq, xs = oracle.quant_rows(x)
    wq, ws = oracle.quant_rows(w)
    y = oracle.linear(xq, xs, wq, ws, 0)
    ref = (x.double() @ w.double().T).numpy()
    rel = np.abs(y - ref).max() / np.abs(ref).max()
    assert rel < 0.05


def test_tiny_config_sampled_outputs_equal_exact_rationals():
    # the tiny 16x256 -> 512 configuration with its synthetic inputs (two
    # outlier input columns), quantized by the oracle: 96 sampled outputs,
    # the first and last included, against exact rationals, in both modes
    M, K, N = 16, 256, 512
    x = synth.make_x(M, K, seed=0, n_out=2)
    w = synth.make_w(N, K, seed=0)
    rng = np.random.default_rng(16)
    pairs = [(0, 0), (M - 1, N - 1)] + [(int(rng.integers(M)), int(rng.integers(N))) for _ in range(94)]
    for mode in (oracle.CHANNEL_TOKEN, oracle.BLOCK128):
        xq, xs = oracle.quant_act(x, mode)
        wq, ws = oracle.quant_weight(w, mode)
        y = oracle.linear(xq, xs, wq, ws, mode)
        sub_m = sorted({m for m, _ in pairs})
        sub_n = sorted({n for _, n in pairs})
        if mode == oracle.CHANNEL_TOKEN:
            ex = _pins.exact_linear_channel(xq[sub_m].tolist(), xs[sub_m], wq[sub_n].tolist(), ws[sub_n])
            for m, n in pairs:
                e = float(ex[sub_m.index(m)][sub_n.index(n)])
                assert abs(float(y[m, n]) - e) <= 0.5 * _pins.f32_ulp(e) * 1.0000001 + 1e-300, (mode, m, n)
        else:
            from fractions import Fraction
            for m, n in pairs:
                e = Fraction(0)
                for kb in range(K // 128):
                    acc = sum(Fraction(float(VALS[xq[m, k]])) * Fraction(float(VALS[wq[n, k]]))
                              for k in range(128 * kb, 128 * kb + 128))
                    e += acc * Fraction(float(xs[m, kb])) * Fraction(float(ws[n // 128, kb]))
                e = float(e)
                assert abs(float(y[m, n]) - e) <= 2 * _pins.f32_ulp(e) + 1e-300, (mode, m, n)
