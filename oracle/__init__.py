"""CPU oracle for the FP8 W8A8 linear layer (ctypes wrapper over fp8_oracle.c).

TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline leg are the only callers.  The GPU product path never imports
this package and must not be routed through it.

Arrays are numpy: bf16 tensors travel as their uint16 bit patterns, codes as
uint8, scales as float32.  See fp8_oracle.c for what each function computes
and which page passage it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CHANNEL_TOKEN = 0
BLOCK128 = 1


# ISO C11 with every warning an error: a compiler that rejects something the
# source relies on (an implicit declaration, say) fails the build, not the tests.
WARN_FLAGS = ["-std=c11", "-Wall", "-Wextra", "-Wpedantic", "-Werror"]


def build(force: bool = False) -> str:
    """Compile fp8_oracle.c into liboracle.so (gcc, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2"] + WARN_FLAGS + ["-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-ffp-contract=off", "-fvisibility=hidden",
               _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int64
        _lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        _lib.orc_e4m3_decode.restype = ctypes.c_double
        _lib.orc_e5m2_decode.argtypes = [ctypes.c_uint8]
        _lib.orc_e5m2_decode.restype = ctypes.c_double
        _lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
        _lib.orc_e4m3_encode.restype = ctypes.c_uint8
        _lib.orc_e4m3_encode_n.argtypes = [P, I, P]
        _lib.orc_e4m3_encode_n.restype = None
        for f in ("orc_quant_rows", "orc_quant_groups128", "orc_quant_blocks128",
                  "orc_quant_rows_s16", "orc_quant_groups128_s16", "orc_quant_blocks128_s16"):
            getattr(_lib, f).argtypes = [P, I, I, I, P, I, P]
            getattr(_lib, f).restype = None
        _lib.orc_linear.argtypes = [P, P, P, P, I, I, I, I, I, ctypes.c_int, P]
        _lib.orc_linear.restype = None
        _lib.orc_linear_at.argtypes = [P, P, P, P, I, I, I, ctypes.c_int, P, P, I, P]
        _lib.orc_linear_at.restype = None
        _lib.orc_linear_w8a16.argtypes = [P, P, P, I, I, I, P]
        _lib.orc_linear_w8a16.restype = None
        _lib.orc_quant_static.argtypes = [P, I, I, I, ctypes.c_float, P, I]
        _lib.orc_quant_static.restype = None
        _lib.orc_linear_swiglu.argtypes = [P, P, P, P, P, P, I, I, I, P]
        _lib.orc_linear_swiglu.restype = None
        _lib.orc_rmsnorm_rstd.argtypes = [P, I, I, I, ctypes.c_float, P]
        _lib.orc_rmsnorm_rstd.restype = None
        _lib.orc_rmsnorm_quant_rows.argtypes = [P, P, I, I, I, ctypes.c_float, ctypes.c_int, P, I, P, P, P]
        _lib.orc_rmsnorm_quant_rows.restype = None
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """bf16 torch tensor or uint16 array -> C-contiguous uint16 numpy array."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        x = x.detach().cpu().contiguous().view(torch.uint16).numpy()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    return x


def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(int(code) & 0xFF)


def e5m2_decode(code: int) -> float:
    return lib().orc_e5m2_decode(int(code) & 0xFF)


def e4m3_encode(v: float) -> int:
    return int(lib().orc_e4m3_encode(float(v)))


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    """Encode each float32 of v (scale 1) through the oracle's encoder."""
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode_n(_p(v), v.size, _p(out))
    return out


def quant_rows(x, scale_bf16: bool = False):
    """One amax/448 scale per row.  x: bf16 [R, K] -> (codes u8 [R, K], scales f32 [R]).
    scale_bf16: round each scale to bf16 before computing the codes."""
    xb = _bits(x)
    R, K = xb.shape
    q = np.empty((R, K), np.uint8)
    s = np.empty((R,), np.float32)
    (lib().orc_quant_rows_s16 if scale_bf16 else lib().orc_quant_rows)(_p(xb), R, K, K, _p(q), K, _p(s))
    return q, s


def linear_w8a16(x, wq, ws) -> np.ndarray:
    """Weight-only FP8: bf16 activations x [M, K] times dequantized codes wq [N, K]
    with per-channel scales ws [N].  -> fp32 [M, N]."""
    xb = _bits(x)
    wq = np.ascontiguousarray(wq, np.uint8)
    ws = np.ascontiguousarray(ws, np.float32)
    M, K = xb.shape
    N = wq.shape[0]
    y = np.empty((M, N), np.float32)
    lib().orc_linear_w8a16(_p(xb), _p(wq), _p(ws), M, N, K, _p(y))
    return y


def linear_swiglu(xq, xs, wq_gate, ws_gate, wq_up, ws_up) -> np.ndarray:
    """bf16(bf16(silu(g)) * u) of the exact gate and up linears (channel/token
    scales), g and u rounded to bf16 first.  -> bf16 bits uint16 [M, N]."""
    xq = np.ascontiguousarray(xq, np.uint8)
    wg = np.ascontiguousarray(wq_gate, np.uint8)
    wu = np.ascontiguousarray(wq_up, np.uint8)
    xs = np.ascontiguousarray(xs, np.float32)
    sg = np.ascontiguousarray(ws_gate, np.float32)
    su = np.ascontiguousarray(ws_up, np.float32)
    M, K = xq.shape
    N = wg.shape[0]
    assert wg.shape == (N, K) and wu.shape == (N, K)
    act = np.empty((M, N), np.uint16)
    lib().orc_linear_swiglu(_p(xq), _p(xs), _p(wg), _p(sg), _p(wu), _p(su), M, N, K, _p(act))
    return act


def rmsnorm_rstd(x, eps: float = 1e-5) -> np.ndarray:
    """Per-row 1 / sqrt(mean(x^2) + eps) in fp32 (exact mean, rounded once)."""
    xb = _bits(x)
    R, K = xb.shape
    r = np.empty((R,), np.float32)
    lib().orc_rmsnorm_rstd(_p(xb), R, K, K, float(eps), _p(r))
    return r


def rmsnorm_quant_rows(x, gamma, eps: float = 1e-5, rstd_ulps: int = 0):
    """RMSNorm of every row with the oracle's own rstd, then one amax/448 scale
    per row.  rstd_ulps moves that rstd by whole fp32 steps before it is used
    (0: the definition; the parity tests also use +-1).
    -> (codes u8 [R, K], scales f32 [R], normalised rows bf16 bits u16 [R, K], rstd f32 [R])."""
    xb = _bits(x)
    gb = _bits(gamma).ravel()
    R, K = xb.shape
    assert gb.size == K
    q = np.empty((R, K), np.uint8)
    s = np.empty((R,), np.float32)
    y = np.empty((R, K), np.uint16)
    r = np.empty((R,), np.float32)
    lib().orc_rmsnorm_quant_rows(_p(xb), _p(gb), R, K, K, float(eps), int(rstd_ulps), _p(q), K, _p(s), _p(y), _p(r))
    return q, s, y, r


def quant_static(x, scale: float) -> np.ndarray:
    """Codes of every element with one fixed scale (no amax).  -> codes u8 [R, K]."""
    xb = _bits(x)
    R, K = xb.shape
    q = np.empty((R, K), np.uint8)
    lib().orc_quant_static(_p(xb), R, K, K, float(scale), _p(q), K)
    return q


def percentile_scale(x, lo: float = 0.001, hi: float = 0.999) -> float:
    """Static scale from a calibration tensor: the larger magnitude of its lo and
    hi quantiles (linear interpolation between order statistics), / 448, in
    fp32.  1.0 when that range is zero."""
    f = np.sort(((_bits(x).astype(np.uint32) << 16).view(np.float32)).astype(np.float64), axis=None)
    def q(p):
        pos = p * (f.size - 1)
        i = int(np.floor(pos))
        j = min(i + 1, f.size - 1)
        return f[i] + (f[j] - f[i]) * (pos - i)
    amax = max(abs(q(lo)), abs(q(hi)))
    return float(np.float32(np.float32(amax) / np.float32(448.0))) if amax > 0 else 1.0


def quant_groups128(x, scale_bf16: bool = False):
    """One scale per 128-group of each row.  -> (codes [M, K], scales [M, K/128])."""
    xb = _bits(x)
    M, K = xb.shape
    assert K % 128 == 0
    q = np.empty((M, K), np.uint8)
    s = np.empty((M, K // 128), np.float32)
    (lib().orc_quant_groups128_s16 if scale_bf16 else lib().orc_quant_groups128)(_p(xb), M, K, K, _p(q), K, _p(s))
    return q, s


def quant_blocks128(w, scale_bf16: bool = False):
    """One scale per 128x128 tile.  -> (codes [N, K], scales [ceil(N/128), K/128])."""
    wb = _bits(w)
    N, K = wb.shape
    assert K % 128 == 0
    q = np.empty((N, K), np.uint8)
    s = np.empty(((N + 127) // 128, K // 128), np.float32)
    (lib().orc_quant_blocks128_s16 if scale_bf16 else lib().orc_quant_blocks128)(_p(wb), N, K, K, _p(q), K, _p(s))
    return q, s


def quant_weight(w, mode: int, scale_bf16: bool = False):
    return quant_rows(w, scale_bf16) if mode == CHANNEL_TOKEN else quant_blocks128(w, scale_bf16)


def quant_act(x, mode: int, scale_bf16: bool = False):
    return quant_rows(x, scale_bf16) if mode == CHANNEL_TOKEN else quant_groups128(x, scale_bf16)


def linear(xq, xs, wq, ws, mode: int) -> np.ndarray:
    """Exact layer output Y [M, N] (fp32) from codes and scales."""
    xq = np.ascontiguousarray(xq, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    xs = np.ascontiguousarray(xs, np.float32)
    ws = np.ascontiguousarray(ws, np.float32)
    M, K = xq.shape
    N = wq.shape[0]
    y = np.empty((M, N), np.float32)
    lib().orc_linear(_p(xq), _p(xs), _p(wq), _p(ws), M, N, K, K, K, mode, _p(y))
    return y


def linear_at(xq, xs, wq, ws, mode: int, ms, ns) -> np.ndarray:
    """Exact outputs Y[ms[i], ns[i]] only."""
    xq = np.ascontiguousarray(xq, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    xs = np.ascontiguousarray(xs, np.float32)
    ws = np.ascontiguousarray(ws, np.float32)
    ms = np.ascontiguousarray(ms, np.int64)
    ns = np.ascontiguousarray(ns, np.int64)
    K = xq.shape[1]
    y = np.empty(ms.shape, np.float32)
    lib().orc_linear_at(_p(xq), _p(xs), _p(wq), _p(ws), K, K, K, mode,
                        _p(ms), _p(ns), ms.size, _p(y))
    return y
