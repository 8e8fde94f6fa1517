"""fp8_linear_noalloc: the small-M linear for callers that cannot allocate.

Some callers cannot allocate device memory when they call (plugin or enqueue
interfaces that provide no scratch, latency-critical code that must not pay
cudaMalloc's implicit synchronisation, fixed memory budgets).  For them
libfp8q.so has one entry point whose split-K scratch is a fixed 16 MiB array
inside the library.  These tests call it through the C ABI and check that it
gives what fp8_linear (with a caller-supplied workspace) gives, within the
tolerance the other parity tests use, on two calls in a row; the second call
finds the first call's leftovers in the shared array.

This file is collected last on purpose and needs nothing from earlier tests.
"""
import ctypes

import pytest
import torch

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
    x = synth.make_x(M, K, seed=seed).to(DEV)
    w = synth.make_w(N, K, seed=seed).to(DEV)
    wq, ws = fq.fp8_quant_weight(w, mode)
    xq, xs = fq.fp8_quant_act(x, mode)
    return xq, xs, wq, ws


def _noalloc(L, xq, xs, wq, ws, mode, N):
    M, K = xq.shape
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    st = L.fp8_linear_noalloc(xq.data_ptr(), xs.data_ptr(), wq.data_ptr(), ws.data_ptr(), M, N, K, mode,
                              y.data_ptr(), y.stride(0), torch.cuda.current_stream().cuda_stream)
    assert st == fq.OK, fq.status_string(st)
    return y


def test_two_calls_in_a_row_match_fp8_linear(L):
    cases = [(16, 8192, 3072, fq.CHANNEL_TOKEN, 1),     # first call fills the scratch
             (5, 2048, 1024, fq.BLOCK128, 2)]          # second call runs over the leftovers
    for (M, N, K, mode, seed) in cases:
        xq, xs, wq, ws = _operands(M, N, K, mode, seed)
        y_new = _noalloc(L, xq, xs, wq, ws, mode, N)
        y_ref = fq.fp8_linear(xq, xs, wq, ws, mode)      # existing entry point, torch workspace
        torch.cuda.synchronize()
        P.assert_y_close(y_new.float().cpu().numpy(), y_ref.float().cpu().numpy(),
                         what=f"noalloc vs fp8_linear M={M} N={N} K={K} mode={mode}")
    assert fq.device_error(clear=True) == 0


def test_rejects_what_it_cannot_serve(L):
    # M > 64 is not its path; a problem whose scratch exceeds 16 MiB is refused.
    # Real buffers, so that a wrong answer could not touch stray memory.
    xq, xs, wq, ws = _operands(65, 256, 256, fq.CHANNEL_TOKEN, 3)
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
