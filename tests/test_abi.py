"""The C-ABI library: it loads, exports every function include/fp8q.h declares,
and rejects bad arguments before touching CUDA (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import fp8_w8a8_quantized_amax_b200 as fq
from fp8_w8a8_quantized_amax_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in os.listdir(os.path.join(ROOT, "include"))
           if h.endswith(".h")]


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*FP8Q_API\s+[^;(]*?\b(fp8\w*)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    fbuild.build()
    return fq.lib()


def test_header_declares_the_three_entry_points():
    d = declared_functions()
    for n in ("fp8_quant_weight", "fp8_quant_act", "fp8_linear"):
        assert n in d


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", fq.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(\w+)", out))
    for n in declared_functions():
        assert n in exported, n
        assert getattr(L, n) is not None


def test_library_exports_nothing_else_public(L):
    out = subprocess.run(["nm", "-D", "--defined-only", fq.LIB_PATH], capture_output=True, text=True).stdout
    ours = {s for s in re.findall(r"\bT\s+(\w+)", out) if s.startswith("fp8")}
    assert ours == set(declared_functions())


def test_status_strings(L):
    for s in range(6):
        assert fq.status_string(s).startswith("FP8Q")
    assert "unknown" in fq.status_string(99)


def test_version(L):
    assert fq.version() >= 100


P = 0x10000          # a 16-byte aligned dummy address (never dereferenced here)
BAD = 0x10001        # misaligned


def q_act(L, x=P, M=4, K=256, ldx=256, mode=0, q=P, ldq=256, s=P):
    return L.fp8_quant_act(x, M, K, ldx, mode, q, ldq, s, None)


def q_w(L, w=P, N=4, K=256, ldw=256, mode=0, q=P, ldq=256, s=P):
    return L.fp8_quant_weight(w, N, K, ldw, mode, q, ldq, s, None)


def lin(L, M=4, N=64, K=256, mode=0, y=P, ldy=64, xq=P, xs=P, wq=P, ws=P, wsp=P, wsb=1 << 30):
    return L.fp8_linear(xq, xs, wq, ws, M, N, K, mode, y, ldy, wsp, wsb, None)


@pytest.mark.parametrize("kw,want", [
    (dict(mode=2), fq.ERR_INVALID_ARG),
    (dict(mode=-1), fq.ERR_INVALID_ARG),
    (dict(K=0), fq.ERR_INVALID_ARG),
    (dict(K=24, ldx=24, ldq=32), fq.ERR_INVALID_ARG),        # K % 16
    (dict(M=-1), fq.ERR_INVALID_ARG),
    (dict(ldx=128), fq.ERR_INVALID_ARG),                     # ld < K
    (dict(ldq=128), fq.ERR_INVALID_ARG),
    (dict(x=None), fq.ERR_INVALID_ARG),
    (dict(q=None), fq.ERR_INVALID_ARG),
    (dict(s=None), fq.ERR_INVALID_ARG),
    (dict(x=BAD), fq.ERR_MISALIGNED),
    (dict(q=P + 8), fq.ERR_MISALIGNED),
    (dict(ldx=260), fq.ERR_MISALIGNED),
    (dict(ldq=264), fq.ERR_MISALIGNED),
    (dict(mode=1, K=192, ldx=192, ldq=192), fq.ERR_INVALID_ARG),   # block mode needs K % 128
    (dict(M=0, x=None, q=None, s=None), fq.OK),              # empty input is a no-op
    (dict(mode=0x12), fq.ERR_INVALID_ARG),                   # the bf16-scale option on an unknown mode
    (dict(mode=0x20), fq.ERR_INVALID_ARG),                   # an unknown option
    (dict(mode=0x11, K=192, ldx=192, ldq=192), fq.ERR_INVALID_ARG),   # block mode with the option: K % 128
    (dict(mode=0x10, M=0, x=None, q=None, s=None), fq.OK),
])
def test_quant_act_argument_checks(L, kw, want):
    assert q_act(L, **kw) == want


def q_static(L, x=P, M=4, K=256, ldx=256, scale=0.05, q=P, ldq=256, s=P):
    return L.fp8_quant_act_static(x, M, K, ldx, scale, q, ldq, s, None)


@pytest.mark.parametrize("kw,want", [
    (dict(scale=0.0), fq.ERR_INVALID_ARG),
    (dict(scale=-1.0), fq.ERR_INVALID_ARG),
    (dict(scale=float("nan")), fq.ERR_INVALID_ARG),
    (dict(scale=float("inf")), fq.ERR_INVALID_ARG),
    (dict(K=24, ldx=24, ldq=32), fq.ERR_INVALID_ARG),
    (dict(M=-1), fq.ERR_INVALID_ARG),
    (dict(x=None), fq.ERR_INVALID_ARG),
    (dict(q=None), fq.ERR_INVALID_ARG),
    (dict(x=BAD), fq.ERR_MISALIGNED),
    (dict(s=P + 2), fq.ERR_MISALIGNED),
    (dict(M=0, x=None, q=None, s=None), fq.OK),
])
def test_quant_static_argument_checks(L, kw, want):
    assert q_static(L, **kw) == want


def swi(L, M=4, N=64, K=256, y=P, ldy=64, xq=P, xs=P, wg=P, sg=P, wu=P, su=P):
    return L.fp8_linear_swiglu(xq, xs, wg, sg, wu, su, M, N, K, y, ldy, None)


@pytest.mark.parametrize("kw,want", [
    (dict(wu=None), fq.ERR_INVALID_ARG),
    (dict(su=None), fq.ERR_INVALID_ARG),
    (dict(wg=None), fq.ERR_INVALID_ARG),
    (dict(K=24), fq.ERR_INVALID_ARG),
    (dict(N=24, ldy=24), fq.ERR_INVALID_ARG),
    (dict(ldy=32), fq.ERR_INVALID_ARG),
    (dict(wu=BAD), fq.ERR_MISALIGNED),
    (dict(su=P + 2), fq.ERR_MISALIGNED),
    (dict(M=0, xq=None, xs=None, wg=None, sg=None, wu=None, su=None, y=None), fq.OK),
])
def test_swiglu_argument_checks(L, kw, want):
    assert swi(L, **kw) == want


def w16(L, x=P, ldx=256, w=P, ws=P, M=4, N=40, K=256, y=P, ldy=40, wk=P, wkb=1 << 30):
    return L.fp8_linear_w8a16(x, ldx, w, ws, M, N, K, y, ldy, wk, wkb, None)


@pytest.mark.parametrize("kw,want", [
    (dict(M=65), fq.ERR_UNSUPPORTED),                       # more than 64 tokens: W8A8 path
    (dict(M=-1), fq.ERR_INVALID_ARG),
    (dict(K=24, ldx=24), fq.ERR_INVALID_ARG),               # K % 16
    (dict(ldx=128), fq.ERR_INVALID_ARG),                    # ldx < K
    (dict(ldy=39), fq.ERR_INVALID_ARG),                     # ldy < N
    (dict(N=0), fq.ERR_INVALID_ARG),
    (dict(w=None), fq.ERR_INVALID_ARG),
    (dict(ws=None), fq.ERR_INVALID_ARG),
    (dict(ldx=260), fq.ERR_MISALIGNED),                     # row starts off 16 bytes
    (dict(x=BAD), fq.ERR_MISALIGNED),
    (dict(w=P + 8), fq.ERR_MISALIGNED),
    (dict(y=P + 1), fq.ERR_MISALIGNED),
    (dict(M=0, x=None, w=None, ws=None, y=None, wk=None, wkb=0), fq.OK),
])
def test_w8a16_argument_checks(L, kw, want):
    assert w16(L, **kw) == want


def test_w8a16_workspace_size(L):
    assert L.fp8_linear_w8a16_workspace_size(1, 8192, 8192) == 0        # one token: CUDA-core kernel, no scratch
    assert L.fp8_linear_w8a16_workspace_size(65, 8192, 8192) == 0       # not served
    assert L.fp8_linear_w8a16_workspace_size(0, 8192, 8192) == 0
    # 2..64 tokens: the same scratch as the FP8 linear of that shape (same
    # decode schedule; both are 0 on a machine without a CUDA device)
    for M in (2, 16, 17, 64):
        assert L.fp8_linear_w8a16_workspace_size(M, 8192, 8192) == L.fp8_linear_workspace_size(M, 8192, 8192, 0)


def rms_q(L, x=P, g=P, M=4, K=256, ldx=256, eps=1e-5, q=P, ldq=256, s=P, r=None):
    return L.fp8_rmsnorm_quant_act(x, g, M, K, ldx, eps, q, ldq, s, r, None)


@pytest.mark.parametrize("kw,want", [
    (dict(K=0), fq.ERR_INVALID_ARG),
    (dict(K=24, ldx=24, ldq=32), fq.ERR_INVALID_ARG),        # K % 16
    (dict(M=-1), fq.ERR_INVALID_ARG),
    (dict(ldx=128), fq.ERR_INVALID_ARG),
    (dict(g=None), fq.ERR_INVALID_ARG),
    (dict(x=None), fq.ERR_INVALID_ARG),
    (dict(s=None), fq.ERR_INVALID_ARG),
    (dict(eps=-1.0), fq.ERR_INVALID_ARG),
    (dict(eps=float("nan")), fq.ERR_INVALID_ARG),
    (dict(eps=float("inf")), fq.ERR_INVALID_ARG),
    (dict(g=BAD), fq.ERR_MISALIGNED),
    (dict(x=BAD), fq.ERR_MISALIGNED),
    (dict(r=P + 2), fq.ERR_MISALIGNED),
    (dict(M=0, x=None, g=None, q=None, s=None), fq.OK),      # empty input is a no-op
])
def test_rmsnorm_quant_argument_checks(L, kw, want):
    assert rms_q(L, **kw) == want


@pytest.mark.parametrize("kw,want", [
    (dict(mode=3), fq.ERR_INVALID_ARG),
    (dict(N=-2), fq.ERR_INVALID_ARG),
    (dict(w=None), fq.ERR_INVALID_ARG),
    (dict(w=BAD), fq.ERR_MISALIGNED),
    (dict(mode=1, K=64, ldw=64, ldq=64), fq.ERR_INVALID_ARG),
    (dict(N=0, w=None, q=None, s=None), fq.OK),
])
def test_quant_weight_argument_checks(L, kw, want):
    assert q_w(L, **kw) == want


@pytest.mark.parametrize("kw,want", [
    (dict(mode=5), fq.ERR_INVALID_ARG),
    (dict(N=0), fq.ERR_INVALID_ARG),
    (dict(N=24, ldy=24), fq.ERR_INVALID_ARG),               # N % 16
    (dict(K=40), fq.ERR_INVALID_ARG),                       # K % 16
    (dict(K=272, mode=1), fq.ERR_INVALID_ARG),              # block: K % 128
    (dict(ldy=32), fq.ERR_INVALID_ARG),                     # ldy < N
    (dict(ldy=68), fq.ERR_MISALIGNED),
    (dict(y=BAD), fq.ERR_MISALIGNED),
    (dict(xq=P + 4), fq.ERR_MISALIGNED),
    (dict(wq=None), fq.ERR_INVALID_ARG),
    (dict(xs=None), fq.ERR_INVALID_ARG),
    (dict(M=-3), fq.ERR_INVALID_ARG),
    (dict(M=0, xq=None, xs=None, wq=None, ws=None, y=None), fq.OK),
    (dict(wsp=None), fq.ERR_INVALID_ARG),                   # M <= 64 needs a workspace
    (dict(wsp=P + 8), fq.ERR_MISALIGNED),                   # workspace: 16-byte alignment
    (dict(wsp=P + 4, M=64), fq.ERR_MISALIGNED),
])
def test_linear_argument_checks(L, kw, want):
    assert lin(L, **kw) == want


def noalloc(L, M=4, N=64, K=256, mode=0, y=P, ldy=64, xq=P, xs=P, wq=P, ws=P):
    f = L.fp8_linear_noalloc
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64] * 3 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_int64,
                                                                 ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f(xq, xs, wq, ws, M, N, K, mode, y, ldy, None)


@pytest.mark.parametrize("kw,want", [
    (dict(M=65), fq.ERR_UNSUPPORTED),                       # the M > 64 path needs no scratch: use fp8_linear
    (dict(mode=5), fq.ERR_INVALID_ARG),
    (dict(K=40), fq.ERR_INVALID_ARG),
    (dict(y=BAD), fq.ERR_MISALIGNED),
    (dict(wq=None), fq.ERR_INVALID_ARG),
    (dict(M=0, xq=None, xs=None, wq=None, ws=None, y=None), fq.OK),
])
def test_noalloc_argument_checks(L, kw, want):
    assert noalloc(L, **kw) == want


def calib(L, x=P, M=4, K=256, ldx=256, lo=0.001, hi=0.999, h=P, s=P):
    return L.fp8_calibrate_static_scale(x, M, K, ldx, lo, hi, h, s, None)


@pytest.mark.parametrize("kw,want", [
    (dict(M=0), fq.ERR_INVALID_ARG),                         # no values: no quantile
    (dict(K=12, ldx=12), fq.ERR_INVALID_ARG),                # K % 8
    (dict(ldx=128), fq.ERR_INVALID_ARG),
    (dict(lo=-0.1), fq.ERR_INVALID_ARG),
    (dict(hi=1.5), fq.ERR_INVALID_ARG),
    (dict(lo=float("nan")), fq.ERR_INVALID_ARG),
    (dict(x=None), fq.ERR_INVALID_ARG),
    (dict(h=None), fq.ERR_INVALID_ARG),
    (dict(s=None), fq.ERR_INVALID_ARG),
    (dict(x=BAD), fq.ERR_MISALIGNED),
    (dict(h=P + 2), fq.ERR_MISALIGNED),
    (dict(ldx=260), fq.ERR_MISALIGNED),
    (dict(M=1 << 20, K=1 << 12, ldx=1 << 12), fq.ERR_UNSUPPORTED),    # 2^32 values
])
def test_calibrate_argument_checks(L, kw, want):
    assert calib(L, **kw) == want


def test_workspace_size_is_zero_for_invalid_or_prefill(L):
    assert L.fp8_linear_workspace_size(0, 64, 256, 0) == 0
    assert L.fp8_linear_workspace_size(128, 64, 256, 0) == 0
    assert L.fp8_linear_workspace_size(4, 64, 256, 9) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="needs a machine without a CUDA device")
def test_valid_arguments_without_a_gpu_report_cuda_error(L):
    assert q_act(L) == fq.ERR_CUDA
    assert q_w(L) == fq.ERR_CUDA
    assert lin(L) == fq.ERR_CUDA
    assert lin(L, wsp=P + 16) == fq.ERR_CUDA            # 16-byte alignment is enough
    assert lin(L, M=65, wsp=None, wsb=0) == fq.ERR_CUDA  # the prefill path needs no workspace
    assert noalloc(L) == fq.ERR_CUDA
    assert calib(L) == fq.ERR_CUDA
    assert rms_q(L) == fq.ERR_CUDA
    assert swi(L) == fq.ERR_CUDA
    assert q_static(L) == fq.ERR_CUDA
    assert q_static(L, s=None) == fq.ERR_CUDA           # x_scale is optional
    assert w16(L) == fq.ERR_CUDA
    assert w16(L, N=41, ldy=41, y=P + 2) == fq.ERR_CUDA    # any N; bf16 output alignment only
    assert w16(L, M=1, wk=None, wkb=0) == fq.ERR_CUDA      # one token needs no workspace


def test_binding_refuses_cpu_tensors(L):
    with pytest.raises(ValueError):
        fq.fp8_quant_act(torch.zeros(4, 256, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        fq.fp8_quant_weight(torch.zeros(4, 256, dtype=torch.bfloat16))
