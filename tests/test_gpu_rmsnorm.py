"""GPU fused RMSNorm + per-token quantization vs the oracle.

The oracle computes everything itself from the definition: the exact mean
of squares rounded once to fp32, the correctly rounded 1/sqrt(ms + eps), then
the bf16 normalisation and the per-token quantization.  Nothing the kernel
computed is passed to it.

The kernel sums the (exact) squares in fp64, so its mean of squares is the
exactly rounded one except for a mean within a few fp64 roundings of an fp32
rounding boundary, where it can be one fp32 step off, and rstd with it.  So:
rows whose rstd equals the oracle's must have bit-identical codes and scales;
a row whose rstd is one fp32 step off must have the codes and scales of the
oracle run with its rstd moved by that step (the oracle's rstd_ulps knob);
no row may be further off; and the fraction of rows with an equal rstd is
reported and must be at least 99%.
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


def check(x, g, eps=1e-5, rows=None, min_equal=0.99):
    q, s, r = fq.fp8_rmsnorm_quant_act(x.to(DEV), g.to(DEV), eps, return_rstd=True)
    xc = x.cpu() if rows is None else x.cpu()[torch.as_tensor(rows)]
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.as_tensor(rows, device=t.device)])
    q_g, s_g, r_g = (sel(t).cpu().numpy() for t in (q, s, r))
    ref_q, ref_s, _, ref_r = oracle.rmsnorm_quant_rows(xc, g, eps=eps)
    # positive fp32 values order like their bit patterns: the difference of
    # the patterns counts fp32 steps
    d = r_g.view(np.int32).astype(np.int64) - ref_r.view(np.int32).astype(np.int64)
    assert np.all(np.abs(d) <= 1), f"rstd off by {np.abs(d).max()} fp32 steps"
    for u in (-1, 0, 1):
        m = d == u
        if not m.any():
            continue
        if u == 0:
            uq, us = ref_q[m], ref_s[m]
        else:   # the oracle on those rows alone, its rstd moved by u
            uq, us, _, _ = oracle.rmsnorm_quant_rows(xc[torch.from_numpy(m)], g, eps=eps, rstd_ulps=u)
        P.assert_codes_equal(torch.from_numpy(q_g[m]), uq, f"rmsnorm codes {tuple(x.shape)}, rstd {u:+d}")
        P.assert_scales_equal(torch.from_numpy(s_g[m]), us, f"rmsnorm scales {tuple(x.shape)}, rstd {u:+d}")
    frac = float((d == 0).mean())
    print(f"rmsnorm {tuple(x.shape)} eps={eps}: rstd equal to the oracle's on {frac:.4%} of {d.size} rows")
    assert frac >= min_equal, f"rstd equal on only {frac:.4%} of rows"
    # without the rstd output: the same codes
    q2, s2 = fq.fp8_rmsnorm_quant_act(x.to(DEV), g.to(DEV), eps)
    assert torch.equal(q2, q) and torch.equal(s2, s)
    return frac


@pytest.mark.parametrize("M,K", [(1, 16), (3, 48), (17, 3072), (5, 4096), (129, 8192), (2, 1040), (3, 65536)])
def test_rmsnorm_quant_vs_oracle(M, K):
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
    # (the oracle's own normalised rows), on every row where the rstd agree
    x = synth.make_x(64, 4096, seed=8)
    g = _gamma(4096, seed=8)
    q, s, r = fq.fp8_rmsnorm_quant_act(x.to(DEV), g.to(DEV), return_rstd=True)
    _, _, y, r0 = oracle.rmsnorm_quant_rows(x, g)
    same = torch.from_numpy(r.cpu().numpy() == r0)
    assert same.float().mean() >= 0.99
    yt = torch.from_numpy(y.astype(np.int16)).view(torch.bfloat16).to(DEV)
    q2, s2 = fq.fp8_quant_act(yt, fq.CHANNEL_TOKEN)
    same = same.to(DEV)
    assert torch.equal(q[same], q2[same]) and torch.equal(s[same], s2[same])


@pytest.mark.parametrize("M,K", [(8192, 4096), (8192, 8192), (2048, 3072)])
def test_rmsnorm_full_size(M, K):
    # the activations that follow an RMSNorm at the Llama-3.1-8B / -70B and
    # -3.2-3B workload shapes, every row compared
    x = synth.make_x_device(M, K, seed=12)
    check(x, _gamma(K, seed=12))


def test_rmsnorm_empty():
    x = torch.empty(0, 256, dtype=torch.bfloat16, device=DEV)
    q, s = fq.fp8_rmsnorm_quant_act(x, torch.ones(256, dtype=torch.bfloat16, device=DEV))
    assert q.shape == (0, 256) and s.shape == (0,)
