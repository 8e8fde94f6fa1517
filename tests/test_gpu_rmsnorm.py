"""GPU fused RMSNorm + per-token quantization vs the oracle.

The only step the definition leaves open is the order of the fp32 sum of
squares.  So rstd is checked against the oracle's (exact mean, rounded once)
within the error bound of an fp32 sum.  The kernel sums at most 8 * 16 = 128
squares per thread, then over 32 lanes and at most 32 warps, so the bound is
(128 + 5 + 5) roundings of 2^-24 on the mean.  The division by K, the eps
addition and the correctly rounded rsqrt add at most 2.5 ulp; rstd sees half
the mean's relative error.  Given the GPU's rstd, the normalised rows, codes
and scales are exact, and the oracle must reproduce them bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import fp8_w8a8_quantized_amax_b200 as fq
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"
RSTD_REL_BOUND = (0.5 * (128 + 5 + 5) + 2.5) * 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _built():
    from fp8_w8a8_quantized_amax_b200 import build
    build.build()
    fq.device_error(clear=True)
    yield
    assert fq.device_error(clear=True) == 0


def _gamma(K, seed=0):
    g = torch.Generator().manual_seed(seed)
    return (1.0 + 0.1 * torch.randn(K, generator=g)).to(torch.bfloat16)


def check(x, g, eps=1e-5, rows=None):
    q, s, r = fq.fp8_rmsnorm_quant_act(x.to(DEV), g.to(DEV), eps, return_rstd=True)
    xc = x.cpu() if rows is None else x.cpu()[torch.as_tensor(rows)]
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.as_tensor(rows, device=t.device)])
    r_gpu = sel(r).cpu().numpy()
    r_ref = oracle.rmsnorm_rstd(xc, eps)
    rel = np.abs(r_gpu.astype(np.float64) / r_ref.astype(np.float64) - 1.0)
    assert rel.max() <= RSTD_REL_BOUND, f"rstd off by {rel.max():.3g} (bound {RSTD_REL_BOUND:.3g})"
    rq, rs, _, _ = oracle.rmsnorm_quant_rows(xc, g, rstd=r_gpu, eps=eps)
    P.assert_codes_equal(sel(q), rq, f"rmsnorm codes {tuple(x.shape)}")
    P.assert_scales_equal(sel(s), rs, f"rmsnorm scales {tuple(x.shape)}")
    # without the rstd output: the same codes
    q2, s2 = fq.fp8_rmsnorm_quant_act(x.to(DEV), g.to(DEV), eps)
    assert torch.equal(q2, q) and torch.equal(s2, s)


@pytest.mark.parametrize("M,K", [(1, 16), (3, 48), (17, 3072), (5, 4096), (129, 8192), (2, 1040), (3, 65536)])
def test_rmsnorm_quant_bit_exact_given_rstd(M, K):
    check(synth.make_x(M, K, seed=M + K), _gamma(K, seed=K))


def test_rmsnorm_eps_values():
    x = synth.make_x(4, 3072, seed=1)
    for eps in (0.0, 1e-6, 1e-5, 1e-2):
        check(x, _gamma(3072, seed=1), eps)


def test_rmsnorm_special_rows():
    K = 512
    x = torch.zeros(5, K, dtype=torch.bfloat16)
    x[1] = 3.0                                   # constant row
    x[2, 7] = -2.0 ** -60                        # one tiny value
    x[3] = synth.make_x(1, K, seed=3)[0] * 1e6   # large values
    x[4, ::2] = 1.0
    x[4, 1::2] = -1.0
    check(x, _gamma(K, seed=5))


def test_rmsnorm_strided_input_and_output():
    M, K = 37, 4096
    big = synth.make_x(M, 4096 + 256, seed=6).to(DEV)
    x = big[:, 128:128 + K]
    g = _gamma(K, seed=6).to(DEV)
    qbuf = torch.full((M, K + 64), 0xAB, dtype=torch.uint8, device=DEV)
    s = torch.empty(M, dtype=torch.float32, device=DEV)
    fq.fp8_rmsnorm_quant_act(x, g, out=(qbuf[:, :K], s))
    q_ref, s_ref = fq.fp8_rmsnorm_quant_act(x.contiguous(), g)
    assert torch.equal(qbuf[:, :K], q_ref) and torch.equal(s, s_ref)
    assert torch.all(qbuf[:, K:] == 0xAB)


def test_rmsnorm_quant_equals_quant_of_the_normalised_rows():
    # the fused op gives what fp8_quant_act gives on the bf16 RMSNorm output
    # (the oracle's rows for the GPU's rstd)
    x = synth.make_x(64, 4096, seed=8)
    g = _gamma(4096, seed=8)
    q, s, r = fq.fp8_rmsnorm_quant_act(x.to(DEV), g.to(DEV), return_rstd=True)
    _, _, y, _ = oracle.rmsnorm_quant_rows(x, g, rstd=r.cpu().numpy())
    yt = torch.from_numpy(y.astype(np.int16)).view(torch.bfloat16).to(DEV)
    q2, s2 = fq.fp8_quant_act(yt, fq.CHANNEL_TOKEN)
    assert torch.equal(q, q2) and torch.equal(s, s2)


@pytest.mark.parametrize("M,K", [(8192, 4096), (8192, 8192), (2048, 3072)])
def test_rmsnorm_full_size_sampled(M, K):
    x = synth.make_x_device(M, K, seed=12)
    rng = np.random.default_rng(0)
    rows = sorted(set([0, M - 1]) | set(rng.integers(0, M, 24).tolist()))
    check(x, _gamma(K, seed=12), rows=rows)


def test_rmsnorm_empty():
    x = torch.empty(0, 256, dtype=torch.bfloat16, device=DEV)
    q, s = fq.fp8_rmsnorm_quant_act(x, torch.ones(256, dtype=torch.bfloat16, device=DEV))
    assert q.shape == (0, 256) and s.shape == (0,)
