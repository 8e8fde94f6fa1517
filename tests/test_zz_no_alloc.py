"""fp8_linear_noalloc: the small-M linear for callers that cannot allocate.

Some callers cannot allocate device memory when they call (plugin or enqueue
interfaces that provide no scratch, latency-critical code that must not pay
cudaMalloc's implicit synchronisation, fixed memory budgets).  For them
libfp8q.so has one entry point whose split-K scratch is a fixed 16 MiB array
inside the library.  These tests call it through the C ABI and check that it
gives bit for bit what fp8_linear (with a caller-supplied workspace) gives --
the same kernels in the same order -- and that both are within the parity
tolerance of the oracle, on calls in a row: each call finds the previous
call's layout in the shared array (the in-kernel split sums, the separate
reduction kernel in channel and in block mode, then the first shape again).

This file is collected last on purpose and needs nothing from earlier tests.
"""
import ctypes

import pytest
import torch

import oracle
import synth
import fp8_w8a8_quantized_amax_b200 as fq
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def L():
    from fp8_w8a8_quantized_amax_b200 import build
    build.build()
    lib = fq.lib()
    f = lib.fp8_linear_noalloc
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64] * 3 + [ctypes.c_int, ctypes.c_void_p,
                                                                  ctypes.c_int64, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return lib


def _operands(M, N, K, mode, seed):
    x = synth.make_x(M, K, seed=seed)
    w = synth.make_w(N, K, seed=seed)
    wq, ws = fq.fp8_quant_weight(w.to(DEV), mode)
    xq, xs = fq.fp8_quant_act(x.to(DEV), mode)
    rxq, rxs = oracle.quant_act(x, mode)
    rwq, rws = oracle.quant_weight(w, mode)
    P.assert_codes_equal(xq, rxq, "x codes")
    P.assert_codes_equal(wq, rwq, "w codes")
    P.assert_scales_equal(xs, rxs, "x scales")
    P.assert_scales_equal(ws, rws, "w scales")
    return (xq, xs, wq, ws), oracle.linear(rxq, rxs, rwq, rws, mode)


def _noalloc(L, xq, xs, wq, ws, mode, N):
    M, K = xq.shape
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    st = L.fp8_linear_noalloc(xq.data_ptr(), xs.data_ptr(), wq.data_ptr(), ws.data_ptr(), M, N, K, mode,
                              y.data_ptr(), y.stride(0), torch.cuda.current_stream().cuda_stream)
    assert st == fq.OK, fq.status_string(st)
    return y


def test_calls_in_a_row_match_fp8_linear_and_the_oracle(L):
    cases = [(16, 8192, 3072, fq.CHANNEL_TOKEN, 1),     # first call: split tiles summed in the GEMM kernel
             (5, 2048, 1024, fq.BLOCK128, 2),          # over its leftovers: the separate reduction kernel
             (48, 2048, 1024, fq.CHANNEL_TOKEN, 3),    # 16 tiles on 128 CTAs: channel mode's reduction kernel
             (16, 8192, 3072, fq.CHANNEL_TOKEN, 1)]    # the first shape again, over all of them
    for (M, N, K, mode, seed) in cases:
        (xq, xs, wq, ws), y_ref = _operands(M, N, K, mode, seed)
        y_new = _noalloc(L, xq, xs, wq, ws, mode, N)
        y_old = fq.fp8_linear(xq, xs, wq, ws, mode)      # existing entry point, torch workspace
        torch.cuda.synchronize()
        what = f"noalloc M={M} N={N} K={K} mode={mode}"
        assert torch.equal(y_new.view(torch.int16), y_old.view(torch.int16)), what + ": differs from fp8_linear"
        P.assert_y_close(y_new.float().cpu().numpy(), y_ref, what=what + " vs the oracle")
    assert fq.device_error(clear=True) == 0


def test_rejects_what_it_cannot_serve(L):
    # M > 64 is not its path; a problem whose scratch exceeds 16 MiB is refused.
    # Real buffers, so that a wrong answer could not touch stray memory.
    (xq, xs, wq, ws), _ = _operands(65, 256, 256, fq.CHANNEL_TOKEN, 3)
    y = torch.empty((65, 256), dtype=torch.bfloat16, device=DEV)
    st = L.fp8_linear_noalloc(xq.data_ptr(), xs.data_ptr(), wq.data_ptr(), ws.data_ptr(), 65, 256, 256, 0,
                              y.data_ptr(), 256, None)
    assert st == fq.ERR_UNSUPPORTED
    M, N, K = 64, 1 << 18, 128                    # (2048 tiles + SMs) x 64 x 512 B > 16 MiB
    xq = torch.zeros((M, K), dtype=torch.uint8, device=DEV)
    xs = torch.ones(M, dtype=torch.float32, device=DEV)
    wq = torch.zeros((N, K), dtype=torch.uint8, device=DEV)
    ws = torch.ones(N, dtype=torch.float32, device=DEV)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    st = L.fp8_linear_noalloc(xq.data_ptr(), xs.data_ptr(), wq.data_ptr(), ws.data_ptr(), M, N, K, 0,
                              y.data_ptr(), N, None)
    assert st == fq.ERR_UNSUPPORTED
