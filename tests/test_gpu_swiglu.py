"""GPU gate/up GEMM with the SiLU * up epilogue vs the oracle.

Tolerance, derived from the GEMM's: the kernel's bf16 gate and up outputs g',
u' are within t_g = 4e-3 max|g| + ulp(g) (and t_u alike) of the exact linears
g, u, the same bound the plain GEMM parity tests hold.  With |silu'| <= 1.1,
  |act' - act| <= 1.1 t_g (|u| + t_u) + (|silu(g)| + 1.1 t_g) t_u
                 + ulp(silu(g)) (|u| + t_u) + ulp(act)
(the last two terms: bf16 roundings of silu and of the product).
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


def _bf16_np(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def _silu(v):
    return v / (1.0 + np.exp(-v))


def run(M, N, K, seed, rows=None):
    x = synth.make_x(M, K, seed=seed)
    wg = synth.make_w(N, K, seed=seed)
    wu = synth.make_w(N, K, seed=seed + 7)
    xq, xs = fq.fp8_quant_act(x.to(DEV))
    gq, gs = fq.fp8_quant_weight(wg.to(DEV))
    uq, us = fq.fp8_quant_weight(wu.to(DEV))
    # the codes and scales the GEMM consumes are first checked against the
    # oracle's own quantization of the same bf16 tensors
    for (q, s), t, what in (((xq, xs), x, "x"), ((gq, gs), wg, "w_gate"), ((uq, us), wu, "w_up")):
        rq, rs = oracle.quant_rows(t)
        P.assert_codes_equal(q, rq, f"swiglu {what} codes")
        P.assert_scales_equal(s, rs, f"swiglu {what} scales")
    act = fq.fp8_linear_swiglu(xq, xs, gq, gs, uq, us)
    return act, (xq, xs, gq, gs, uq, us)


def check_vs_oracle(act, ops, rows=None):
    xq, xs, gq, gs, uq, us = (t.cpu().numpy() for t in ops)
    if rows is not None:
        xq, xs = xq[rows], xs[rows]
        act = act[torch.as_tensor(rows, device=act.device)]
    ref_bits = oracle.linear_swiglu(xq, xs, gq, gs, uq, us)
    ref = torch.from_numpy(ref_bits.astype(np.int16)).view(torch.bfloat16).double().numpy()
    g = oracle.linear(xq, xs, gq, gs, 0).astype(np.float64)
    u = oracle.linear(xq, xs, uq, us, 0).astype(np.float64)
    tg = 4e-3 * np.abs(g).max() + P.bf16_ulp(g)
    tu = 4e-3 * np.abs(u).max() + P.bf16_ulp(u)
    s = _silu(g)
    tol = 1.1 * tg * (np.abs(u) + tu) + (np.abs(s) + 1.1 * tg) * tu + P.bf16_ulp(s) * (np.abs(u) + tu) \
        + P.bf16_ulp(ref)
    err = np.abs(_bf16_np(act) - ref)
    bad = err > tol
    assert not bad.any(), f"{bad.sum()} of {bad.size} out of tolerance; worst excess {np.max(err - tol):.3g}"


@pytest.mark.parametrize("M,N,K", [
    (300, 256, 512),      # two 256-token tiles, the second mostly past M
    (256, 384, 1024),     # three 128-channel tiles
    (1000, 1040, 512),    # ragged M and N (N % 128 = 16)
    (65, 128, 256),       # small M on the pair schedule
    (2048, 2560, 256),    # 160 tiles > pairs: persistent loop, tail split into 64-channel halves
])
def test_swiglu_vs_oracle(M, N, K):
    act, ops = run(M, N, K, seed=M + N)
    check_vs_oracle(act, ops)


def test_swiglu_full_size_sampled():
    # Llama-3.2-3B MLP: M=2048, K=3072, N=8192
    M, N, K = 2048, 8192, 3072
    act, ops = run(M, N, K, seed=3)
    rng = np.random.default_rng(0)
    rows = np.array(sorted(set([0, M - 1]) | set(rng.integers(0, M, 14).tolist())))
    check_vs_oracle(act, ops, rows=rows)


def test_swiglu_agrees_with_the_separate_linears():
    # g and u are fp8_linear's outputs; the only difference to silu(g) * u
    # computed from them on the host (exact silu) is the device exponential,
    # which may move silu's bf16 rounding by one ulp in rare elements
    M, N, K = 512, 1024, 1024
    act, (xq, xs, gq, gs, uq, us) = run(M, N, K, seed=11)
    g = _bf16_np(fq.fp8_linear(xq, xs, gq, gs))
    u = _bf16_np(fq.fp8_linear(xq, xs, uq, us))
    sb = torch.from_numpy(_silu(g)).to(torch.bfloat16).double().numpy()
    ref = torch.from_numpy(sb * u).to(torch.bfloat16).double().numpy()
    a = _bf16_np(act)
    diff = a != ref
    assert diff.mean() < 1e-3, f"{diff.sum()} of {diff.size} differ"
    assert np.all(np.abs(a - ref)[diff] <= (P.bf16_ulp(sb) * np.abs(u) + P.bf16_ulp(ref))[diff])
