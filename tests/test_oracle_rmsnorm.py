"""Pins of the oracle's RMSNorm + per-token quantization.

Llama 3 normalises with RMSNorm (eps = 1e-5) before attention and the MLP
("Llama 3 精读实录", section 1.3) and keeps it in BF16 (section 5), so the
activations the q/k/v and gate/up projections quantize are RMSNorm outputs.
The oracle is checked against exact arithmetic (the mean of squares as a
Python rational, rounded once to fp32; the reciprocal square root from mpmath
at 200 bits, rounded once), against float64 references computed here by torch
(the mean of squares, torch.nn.functional.rms_norm) and against properties
that hold exactly: power-of-two invariance, zero and constant rows, gamma
scaling.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _pins


def _gamma(K, seed=0):
    g = torch.Generator().manual_seed(seed)
    return (1.0 + 0.1 * torch.randn(K, generator=g)).to(torch.bfloat16)


def _bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("M,K,eps", [(5, 3072, 1e-5), (3, 4096, 1e-5), (2, 8192, 1e-6), (4, 16, 1e-5)])
def test_rstd_is_the_rounded_reciprocal_rms(M, K, eps):
    x = synth.make_x(M, K, seed=K)
    r = oracle.rmsnorm_rstd(x, eps)
    ms = (x.double() ** 2).mean(dim=1)
    ms32 = ms.float()                                     # exact mean, rounded to fp32
    d = (ms32 + torch.tensor(eps, dtype=torch.float32))   # fp32 addition
    ref = (1.0 / torch.sqrt(d.double())).float().numpy()
    ulps = np.abs(r.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1, f"rstd differs by {ulps.max()} ulp"


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("K,eps", [(16, 1e-5), (3072, 1e-5), (4096, 1e-6), (8192, 1e-5), (1040, 0.0),
                                   (65536, 1e-5)])
def test_rstd_is_exactly_rounded(K, eps):
    # ms: the exact rational mean of squares (Python integers) rounded once to
    # fp32; rstd: 1/sqrt of fl32(ms + eps) from mpmath, rounded once
    x = synth.make_x(3, K, seed=K + 1)
    r = oracle.rmsnorm_rstd(x, eps)
    b = _bits(x)
    for i in range(3):
        assert r[i] == _pins.rmsnorm_rstd_exact(b[i], eps), f"row {i}"


def test_rstd_exact_on_special_rows():
    K = 512
    rows = torch.zeros(7, K, dtype=torch.bfloat16)
    rows[0] = synth.make_x(1, K, seed=1)[0] * 2.0 ** -70    # squares below fp32's normal range
    rows[1, 3] = 2.0 ** -133                                 # the smallest bf16 subnormal
    rows[1, 9] = 1.5 * 2.0 ** -127                           # a bf16 subnormal
    rows[2] = synth.make_x(1, K, seed=2)[0] * 2.0 ** 40      # large squares
    rows[3, ::3] = 3.0                                       # a third of the row constant
    rows[4] = synth.make_x(1, K, seed=4)[0]
    rows[4, 17] = 2.0 ** 30                                  # one value dominating the sum
    rows[5] = 1.0                                            # mean of squares exactly 1
    b = _bits(rows)
    for eps in (0.0, 1e-5):
        r = oracle.rmsnorm_rstd(rows, eps)
        for i in range(7):
            ms = _pins.f32_nearest(_pins.bf16_bits_sum_of_squares(b[i]) / K)
            if eps == 0.0 and ms == 0:
                assert r[i] == np.inf, f"row {i}: mean of squares rounds to 0, rstd = 1/sqrt(0)"
                continue
            assert r[i] == _pins.rmsnorm_rstd_exact(b[i], eps), f"row {i} eps {eps}"
    # mean of squares 1 and eps 0: rstd exactly 1
    assert oracle.rmsnorm_rstd(rows[5:6], 0.0)[0] == 1.0


def test_rstd_ulps_moves_rstd_by_whole_steps():
    x = synth.make_x(4, 256, seed=5)
    g = _gamma(256, seed=5)
    _, _, _, r0 = oracle.rmsnorm_quant_rows(x, g)
    for u in (-1, 1, 3):
        _, _, _, ru = oracle.rmsnorm_quant_rows(x, g, rstd_ulps=u)
        assert np.array_equal(ru.view(np.int32) - r0.view(np.int32), np.full(4, u, np.int32))


@pytest.mark.parametrize("M,K", [(6, 3072), (3, 4096), (2, 8192)])
def test_normalised_rows_match_rms_norm(M, K):
    x = synth.make_x(M, K, seed=M + K)
    g = _gamma(K, seed=K)
    _, _, y, _ = oracle.rmsnorm_quant_rows(x, g, eps=1e-5)
    ref = torch.nn.functional.rms_norm(x.double(), (K,), weight=g.double(), eps=1e-5)
    yt = _bf16(y).double()
    # two roundings to bf16 (h, then gamma * h): each within 2^-8 relative
    assert torch.all((yt - ref).abs() <= 2.0 ** -7 * ref.abs() * 1.001 + 1e-30)
    # and on average far inside that bound
    assert ((yt - ref).abs() / ref.abs().clamp_min(1e-6)).mean() < 2.0 ** -9


def test_power_of_two_invariance_without_eps():
    x = synth.make_x(4, 3072, seed=9)
    g = _gamma(3072, seed=9)
    q0, s0, y0, _ = oracle.rmsnorm_quant_rows(x, g, eps=0.0)
    for k in (-6, 3, 11):
        xs = (x.float() * 2.0 ** k).to(torch.bfloat16)      # exact: a power of two
        q1, s1, y1, _ = oracle.rmsnorm_quant_rows(xs, g, eps=0.0)
        assert np.array_equal(y0, y1) and np.array_equal(q0, q1) and np.array_equal(s0, s1)


def test_gamma_power_of_two_scales_output_exactly():
    x = synth.make_x(3, 4096, seed=2)
    g = _gamma(4096, seed=2)
    q0, s0, y0, _ = oracle.rmsnorm_quant_rows(x, g)
    q1, s1, y1, _ = oracle.rmsnorm_quant_rows(x, (g.float() * 4.0).to(torch.bfloat16))
    assert torch.equal(_bf16(y1).float(), _bf16(y0).float() * 4.0)
    assert np.array_equal(q0, q1) and np.array_equal(s1, s0 * np.float32(4.0))


def test_zero_and_constant_rows():
    K = 256
    x = torch.zeros(3, K, dtype=torch.bfloat16)
    x[1] = 3.0
    x[2] = -0.5
    g = torch.ones(K, dtype=torch.bfloat16)
    q, s, y, r = oracle.rmsnorm_quant_rows(x, g)
    # zero row: rstd = 1/sqrt(eps), output 0, scale 1, codes 0
    assert r[0] == np.float32(1.0 / np.sqrt(np.float64(np.float32(1e-5))))
    assert s[0] == 1.0 and np.all(q[0] == 0) and np.all(y[0] == 0)
    # constant rows: every element is the row's amax -> +-448 codes
    assert np.all(q[1] == 0x7E) and np.all(q[2] == 0xFE)
    # |y| = bf16(bf16(|c| * rstd)) just below 1 (eps), scale |y| / 448
    for i in (1, 2):
        yv = float(_bf16(y[i : i + 1, :1]).float())
        assert 0.99 < abs(yv) <= 1.0
        assert s[i] == np.float32(np.float32(abs(yv)) / np.float32(448.0))


def test_quantized_rows_follow_the_row_quantizer():
    # the codes and scales of the normalised rows are those of the per-token
    # quantizer (itself pinned against torch's float8 cast): checked here
    # through an independent argmin encoder of y / s
    x = synth.make_x(3, 3072, seed=5)
    g = _gamma(3072, seed=5)
    q, s, y, _ = oracle.rmsnorm_quant_rows(x, g)
    yf = _bf16(y).float().numpy()
    quot = (yf / s[:, None]).astype(np.float32)
    assert np.array_equal(q.ravel(), _pins.encode_argmin(quot.ravel()))
