"""Pins of the oracle's gate/up linears with the SiLU * up activation.

The Llama MLP multiplies SiLU(gate) by up ("Llama 3 精读实录", section 1.3).
The oracle's act = bf16(bf16(silu(g)) * u) over bf16 g and u is checked
against a composition built here from independently pinned parts: the
oracle's exact linear (pinned against rationals), torch's bf16 rounding, and
torch's float64 SiLU.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def _case(M, N, K, seed):
    x = synth.make_x(M, K, seed=seed)
    wg = synth.make_w(N, K, seed=seed)
    wu = synth.make_w(N, K, seed=seed + 7)
    xq, xs = oracle.quant_rows(x)
    gq, gs = oracle.quant_rows(wg)
    uq, us = oracle.quant_rows(wu)
    return xq, xs, gq, gs, uq, us


def _compose(xq, xs, gq, gs, uq, us):
    g = torch.from_numpy(oracle.linear(xq, xs, gq, gs, 0)).to(torch.bfloat16)
    u = torch.from_numpy(oracle.linear(xq, xs, uq, us, 0)).to(torch.bfloat16)
    s = torch.nn.functional.silu(g.double()).to(torch.bfloat16)
    return (s * u).view(torch.int16).numpy().view(np.uint16)      # bf16 * bf16 -> bf16


@pytest.mark.parametrize("M,N,K,seed", [(4, 64, 256, 0), (3, 130, 512, 1), (16, 512, 256, 2)])
def test_swiglu_matches_composition(M, N, K, seed):
    parts = _case(M, N, K, seed)
    act = oracle.linear_swiglu(*parts)
    ref = _compose(*parts)
    assert np.array_equal(act, ref), f"{int((act != ref).sum())} of {act.size} differ"


def test_swiglu_zero_gate_or_up_gives_zero():
    xq, xs, gq, gs, uq, us = _case(3, 64, 256, 3)
    act = oracle.linear_swiglu(xq, xs, np.zeros_like(gq), gs, uq, us)    # g = 0 -> silu = 0
    assert np.all((act & 0x7FFF) == 0)
    act = oracle.linear_swiglu(xq, xs, gq, gs, np.zeros_like(uq), us)    # u = 0
    assert np.all((act & 0x7FFF) == 0)


def test_swiglu_sign_and_large_negative_gate():
    # silu(v) -> v for large v and -> 0 (from below) for very negative v
    xq, xs, gq, gs, uq, us = _case(2, 32, 256, 4)
    big = gs * np.float32(1e4)
    act_pos = oracle.linear_swiglu(xq, xs, gq, big, uq, us)
    g = torch.from_numpy(oracle.linear(xq, xs, gq, big, 0)).to(torch.bfloat16).float()
    u = torch.from_numpy(oracle.linear(xq, xs, uq, us, 0)).to(torch.bfloat16).float()
    a = torch.from_numpy(act_pos.astype(np.int16)).view(torch.bfloat16).float()
    pos = g > 50
    assert torch.allclose(a[pos], (g * u)[pos].to(torch.bfloat16).float(), rtol=2 ** -7, atol=0)
    neg = g < -200
    assert torch.all(a[neg].abs() <= (g.abs() * torch.exp(-g.abs()) * u.abs())[neg] * 2 + 1e-30)
