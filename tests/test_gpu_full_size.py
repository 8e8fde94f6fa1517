"""Every workload at full size: every FP8 code and scale, bit for bit.

For each weight of the five workloads (the tiny case, the Llama-3.2-3B MLP,
the Llama-3.1-8B layer set, the Llama-3.2-3B FP8-Block set and the
Llama-3.1-70B sweep) the GPU's codes and scales of the whole weight, and of
the whole activation of every GEMM that uses it, are compared with the
oracle's own quantization of the same bf16 tensors -- every element, not a
sample.  The layer output of each GEMM is then compared with the oracle's
exact output on every row for decode sizes (M <= 64), else on 30 sampled
rows, and on at least 16 whole 128-row weight blocks spread over N (all of
them when N has fewer), within 4e-3 max|y_ref| + 1 bf16 ulp.  The GEMMs run
through fp8_linear as bench.py runs them (same entry point, workspace from
fp8_linear_workspace_size), so each is checked in the launch configuration
that bench.py times.
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
WORKLOADS = ("tiny_16x256x512", "llama3.2-3b_mlp_m2048", "llama3.1-8b_layer_m8192", "llama3.2-3b_block128",
             "llama3.1-70b_sweep")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from fp8_w8a8_quantized_amax_b200 import build
    build.build()
    fq.device_error(clear=True)
    yield
    assert fq.device_error(clear=True) == 0


def _cases():
    out = []
    for name in WORKLOADS:
        wl = synth.workloads()[name]
        by_w = {}
        for g in wl.gemms:
            by_w.setdefault(g.weight, []).append(g)
        for w, gs in by_w.items():
            out.append(pytest.param(name, w, gs, id=f"{name}:{w}"))
    return out


def _sample(n, k, seed):
    if n <= k:
        return np.arange(n)
    rng = np.random.default_rng(seed)
    return np.array(sorted(set([0, n - 1]) | set(rng.choice(n, k - 2, replace=False).tolist())))


def _assert_quant_equal(q, s, rq, rs, what):
    P.assert_codes_equal(q, rq, what + " codes")
    P.assert_scales_equal(s, rs, what + " scales")


@pytest.mark.parametrize("wl_name,wname,gemms", _cases())
def test_full_size_codes_scales_and_outputs(wl_name, wname, gemms):
    tiny = synth.workloads()[wl_name].tiny
    g0 = gemms[0]
    mode = g0.mode
    w = synth.make_w(g0.N, g0.K, seed=0 if tiny else synth.weight_seed(wname))
    wq, ws = fq.fp8_quant_weight(w.to(DEV), mode)
    rwq, rws = oracle.quant_weight(w, mode)
    _assert_quant_equal(wq, ws, rwq, rws, f"{wl_name} {wname} [{g0.N}x{g0.K}]")
    del w
    for i, g in enumerate(gemms):
        x = synth.make_x(g.M, g.K, seed=i, n_out=2 if tiny else None)
        xq, xs = fq.fp8_quant_act(x.to(DEV), mode)
        rxq, rxs = oracle.quant_act(x, mode)
        _assert_quant_equal(xq, xs, rxq, rxs, f"{wl_name} {g.name} activation [{g.M}x{g.K}]")
        del x
        nws = fq.fp8_linear_workspace_size(g.M, g.N, g.K, mode)
        wsp = torch.zeros(nws, dtype=torch.uint8, device=DEV) if nws else None
        y = fq.fp8_linear(xq, xs, wq, ws, mode, workspace=wsp)
        torch.cuda.synchronize()
        ms = np.arange(g.M) if g.M <= 64 else _sample(g.M, 30, i + 1)
        blocks = _sample(-(-g.N // 128), 16, i + 2)
        ns = np.concatenate([np.arange(b * 128, min(b * 128 + 128, g.N)) for b in blocks])
        sub_ws = rws[ns] if mode == fq.CHANNEL_TOKEN else rws[blocks]
        yref = oracle.linear(rxq[ms], rxs[ms], rwq[ns], sub_ws, mode)
        ygpu = y[torch.as_tensor(ms, device=DEV)][:, torch.as_tensor(ns, device=DEV)].float().cpu().numpy()
        P.assert_y_close(ygpu, yref, what=f"{wl_name} {g.name} M={g.M} K={g.K} N={g.N}")
        del xq, xs, y, wsp
    assert fq.device_error(clear=False) == 0


# GEMMs that share an input, merged over stacked weights (the way bench.py
# also measures them): the stacked per-channel or per-block scales stay
# row-local, so the merged output is the concatenation of the separate ones.
MERGED = [synth.Gemm("gate_up_proj", 2048, 3072, 16384), synth.Gemm("qkv_proj", 8192, 4096, 6144),
          synth.Gemm("gate_up_proj_m16_block", 16, 3072, 16384, synth.BLOCK128)]


@pytest.mark.parametrize("g", MERGED, ids=[g.name for g in MERGED])
def test_merged_shapes(g):
    w = synth.make_w(g.N, g.K, seed=synth.weight_seed(g.name))
    wq, ws = fq.fp8_quant_weight(w.to(DEV), g.mode)
    rwq, rws = oracle.quant_weight(w, g.mode)
    _assert_quant_equal(wq, ws, rwq, rws, g.name + " weight")
    x = synth.make_x(g.M, g.K, seed=5)
    xq, xs = fq.fp8_quant_act(x.to(DEV), g.mode)
    rxq, rxs = oracle.quant_act(x, g.mode)
    _assert_quant_equal(xq, xs, rxq, rxs, g.name + " activation")
    y = fq.fp8_linear(xq, xs, wq, ws, g.mode)
    ms = np.arange(g.M) if g.M <= 64 else _sample(g.M, 30, 1)
    blocks = _sample(g.N // 128, 16, 2)
    ns = np.concatenate([np.arange(b * 128, b * 128 + 128) for b in blocks])
    yref = oracle.linear(rxq[ms], rxs[ms], rwq[ns], rws[ns] if g.mode == 0 else rws[blocks], g.mode)
    ygpu = y[torch.as_tensor(ms, device=DEV)][:, torch.as_tensor(ns, device=DEV)].float().cpu().numpy()
    P.assert_y_close(ygpu, yref, what=g.name)
