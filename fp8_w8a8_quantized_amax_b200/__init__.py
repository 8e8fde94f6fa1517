"""B200 (sm_100a) FP8 W8A8 linear layer: Python binding of libfp8q.so.

The functions here carry the names of the C entry points declared in
include/fp8q.h and only marshal arguments: torch tensors supply device memory
and the current CUDA stream, every step of the computation runs in the
library's CUDA kernels.  There is no CPU fallback; without the built library
(or without a GPU) the calls raise.

    Wq, w_scale = fp8_quant_weight(W, mode)      # once per layer
    Xq, x_scale = fp8_quant_act(X, mode)         # every forward
    Y = fp8_linear(Xq, x_scale, Wq, w_scale, mode)

mode: CHANNEL_TOKEN (per-output-channel weights, per-token activations, the
FP8-Dynamic scheme) or BLOCK128 (128x128 weight blocks, 128-groups of
activations, the FP8-Block scheme).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

from .policy import DEFAULT_IGNORE, should_quantize  # noqa: F401

CHANNEL_TOKEN = 0
BLOCK128 = 1
SCALE_BF16 = 0x10      # option OR'ed into a quantizer's mode: scales rounded to bf16 before the codes

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_MISALIGNED = 3
ERR_CUDA = 4
ERR_DEVICE_TIMEOUT = 5

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8q.so")

_lib = None


class FP8QError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """Load libfp8q.so (built in-tree by build.py); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libfp8q.so not built ({LIB_PATH}); run "
                              "python -m fp8_w8a8_quantized_amax_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
        L.fp8_quant_weight.argtypes = [P, I, I, I, ctypes.c_int, P, I, P, P]
        L.fp8_quant_weight.restype = ctypes.c_int
        L.fp8_quant_act.argtypes = [P, I, I, I, ctypes.c_int, P, I, P, P]
        L.fp8_quant_act.restype = ctypes.c_int
        L.fp8_rmsnorm_quant_act.argtypes = [P, P, I, I, I, ctypes.c_float, P, I, P, P, P]
        L.fp8_rmsnorm_quant_act.restype = ctypes.c_int
        L.fp8_quant_act_static.argtypes = [P, I, I, I, ctypes.c_float, P, I, P, P]
        L.fp8_quant_act_static.restype = ctypes.c_int
        L.fp8_calibrate_static_scale.argtypes = [P, I, I, I, ctypes.c_double, ctypes.c_double, P, P, P]
        L.fp8_calibrate_static_scale.restype = ctypes.c_int
        L.fp8_linear_swiglu.argtypes = [P, P, P, P, P, P, I, I, I, P, I, P]
        L.fp8_linear_swiglu.restype = ctypes.c_int
        L.fp8_linear_w8a16.argtypes = [P, I, P, P, I, I, I, P, I, P, S, P]
        L.fp8_linear_w8a16.restype = ctypes.c_int
        L.fp8_linear_w8a16_workspace_size.argtypes = [I, I, I]
        L.fp8_linear_w8a16_workspace_size.restype = S
        L.fp8_linear.argtypes = [P, P, P, P, I, I, I, ctypes.c_int, P, I, P, S, P]
        L.fp8_linear.restype = ctypes.c_int
        L.fp8_linear_workspace_size.argtypes = [I, I, I, ctypes.c_int]
        L.fp8_linear_workspace_size.restype = S
        L.fp8q_status_string.argtypes = [ctypes.c_int]
        L.fp8q_status_string.restype = ctypes.c_char_p
        L.fp8q_device_error.argtypes = [ctypes.c_int]
        L.fp8q_device_error.restype = ctypes.c_int
        L.fp8q_version.argtypes = []
        L.fp8q_version.restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().fp8q_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != OK:
        raise FP8QError(status, what)


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _require_cuda(t: torch.Tensor, name: str, dtype) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D with unit stride in the last dimension")


def _numel(shape) -> int:
    n = 1
    for d in shape:
        n *= int(d)
    return n


def _require_like(t: Optional[torch.Tensor], name: str, dtype, min_numel: int, ref: torch.Tensor) -> None:
    """A scale vector or scratch buffer handed to a kernel: on ref's CUDA device,
    of `dtype`, contiguous, with at least min_numel elements.  (A host tensor
    would reach the kernel as a host pointer.)"""
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda or t.device != ref.device:
        raise ValueError(f"{name} must be a CUDA tensor on {ref.device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < min_numel:
        raise ValueError(f"{name} has {t.numel()} elements, needs {min_numel}")


def _require_out(t: torch.Tensor, name: str, dtype, shape, ref: torch.Tensor) -> None:
    """An output matrix: on ref's CUDA device, of `dtype` and `shape`, rows with unit stride."""
    if not t.is_cuda or t.device != ref.device:
        raise ValueError(f"{name} must be a CUDA tensor on {ref.device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape) or (t.dim() == 2 and t.stride(1) != 1):
        raise ValueError(f"{name} must be {tuple(shape)} with unit stride in the last dimension")


def scale_shape_weight(N: int, K: int, mode: int) -> Tuple[int, ...]:
    return (N,) if (mode & ~SCALE_BF16) == CHANNEL_TOKEN else ((N + 127) // 128, K // 128)


def scale_shape_act(M: int, K: int, mode: int) -> Tuple[int, ...]:
    return (M,) if (mode & ~SCALE_BF16) == CHANNEL_TOKEN else (M, K // 128)


def fp8_quant_weight(W: torch.Tensor, mode: int = CHANNEL_TOKEN,
                     out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None):
    """W bf16 [N, K] -> (Wq uint8 [N, K] E4M3 codes, w_scale fp32 [N] or [N/128, K/128])."""
    _require_cuda(W, "W", torch.bfloat16)
    N, K = W.shape
    if out is None:
        Wq = torch.empty((N, K), dtype=torch.uint8, device=W.device)
        ws = torch.empty(scale_shape_weight(N, K, mode), dtype=torch.float32, device=W.device)
    else:
        Wq, ws = out
        _require_out(Wq, "Wq", torch.uint8, (N, K), W)
        _require_like(ws, "w_scale", torch.float32, _numel(scale_shape_weight(N, K, mode)), W)
    st = lib().fp8_quant_weight(_ptr(W), N, K, W.stride(0), int(mode), _ptr(Wq), Wq.stride(0),
                                _ptr(ws), _stream(W))
    _check(st, "fp8_quant_weight")
    return Wq, ws


def fp8_quant_act(X: torch.Tensor, mode: int = CHANNEL_TOKEN,
                  out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None):
    """X bf16 [M, K] -> (Xq uint8 [M, K], x_scale fp32 [M] or [M, K/128])."""
    _require_cuda(X, "X", torch.bfloat16)
    M, K = X.shape
    if out is None:
        Xq = torch.empty((M, K), dtype=torch.uint8, device=X.device)
        xs = torch.empty(scale_shape_act(M, K, mode), dtype=torch.float32, device=X.device)
    else:
        Xq, xs = out
        _require_out(Xq, "Xq", torch.uint8, (M, K), X)
        _require_like(xs, "x_scale", torch.float32, _numel(scale_shape_act(M, K, mode)), X)
    st = lib().fp8_quant_act(_ptr(X), M, K, X.stride(0), int(mode), _ptr(Xq), Xq.stride(0),
                             _ptr(xs), _stream(X))
    _check(st, "fp8_quant_act")
    return Xq, xs


def fp8_rmsnorm_quant_act(X: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-5,
                          out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None, return_rstd: bool = False):
    """RMSNorm(X) * gamma in bf16, quantized per token, in one pass.
    X bf16 [M, K], gamma bf16 [K] -> (Xq uint8 [M, K], x_scale fp32 [M][, rstd fp32 [M]])."""
    _require_cuda(X, "X", torch.bfloat16)
    M, K = X.shape
    if not gamma.is_cuda or gamma.device != X.device or gamma.dtype != torch.bfloat16 or gamma.numel() != K \
            or not gamma.is_contiguous():
        raise ValueError("gamma must be a contiguous bf16 CUDA tensor of K elements on X's device")
    if out is None:
        Xq = torch.empty((M, K), dtype=torch.uint8, device=X.device)
        xs = torch.empty((M,), dtype=torch.float32, device=X.device)
    else:
        Xq, xs = out
        _require_out(Xq, "Xq", torch.uint8, (M, K), X)
        _require_like(xs, "x_scale", torch.float32, M, X)
    rstd = torch.empty((M,), dtype=torch.float32, device=X.device) if return_rstd else None
    st = lib().fp8_rmsnorm_quant_act(_ptr(X), _ptr(gamma), M, K, X.stride(0), float(eps), _ptr(Xq), Xq.stride(0),
                                     _ptr(xs), _ptr(rstd), _stream(X))
    _check(st, "fp8_rmsnorm_quant_act")
    return (Xq, xs, rstd) if return_rstd else (Xq, xs)


def fp8_quant_act_static(X: torch.Tensor, scale: float, out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None):
    """X bf16 [M, K] coded with one fixed scale -> (Xq uint8 [M, K], x_scale fp32 [M] filled with scale)."""
    _require_cuda(X, "X", torch.bfloat16)
    M, K = X.shape
    if out is None:
        Xq = torch.empty((M, K), dtype=torch.uint8, device=X.device)
        xs = torch.empty((M,), dtype=torch.float32, device=X.device)
    else:
        Xq, xs = out
        _require_out(Xq, "Xq", torch.uint8, (M, K), X)
        if xs is not None:
            _require_like(xs, "x_scale", torch.float32, M, X)
    st = lib().fp8_quant_act_static(_ptr(X), M, K, X.stride(0), float(scale), _ptr(Xq), Xq.stride(0), _ptr(xs),
                                    _stream(X))
    _check(st, "fp8_quant_act_static")
    return Xq, xs


CALIB_HIST_BINS = 65536


def calibrate_static_scale(X: torch.Tensor, lo: float = 0.001, hi: float = 0.999,
                           hist: Optional[torch.Tensor] = None) -> float:
    """Offline calibration of a static scale (fp8_calibrate_static_scale): the
    larger magnitude of X's lo and hi quantiles, / 448, in fp32; 1.0 for a
    zero range.  X bf16 [M, K] on the GPU.  `hist`: a zero-filled int32
    device buffer of 65536 counts (allocated here when None; left zero)."""
    _require_cuda(X, "X", torch.bfloat16)
    if X.dim() != 2:
        raise ValueError("X must be 2-D [M, K]")
    M, K = X.shape
    if hist is None:
        hist = torch.zeros(CALIB_HIST_BINS, dtype=torch.int32, device=X.device)
    _require_like(hist, "hist", torch.int32, CALIB_HIST_BINS, X)
    scale = torch.empty((), dtype=torch.float32, device=X.device)
    st = lib().fp8_calibrate_static_scale(_ptr(X), M, K, X.stride(0), float(lo), float(hi), _ptr(hist), _ptr(scale),
                                          _stream(X))
    _check(st, "fp8_calibrate_static_scale")
    return float(scale.item())


def fp8_linear_swiglu(Xq: torch.Tensor, x_scale: torch.Tensor, Wq_gate: torch.Tensor, w_scale_gate: torch.Tensor,
                      Wq_up: torch.Tensor, w_scale_up: torch.Tensor,
                      out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """bf16(bf16(silu(g)) * u) of the gate and up projections (channel/token
    scales), g and u never written.  -> Y bf16 [M, N]."""
    _require_cuda(Xq, "Xq", torch.uint8)
    _require_cuda(Wq_gate, "Wq_gate", torch.uint8)
    _require_cuda(Wq_up, "Wq_up", torch.uint8)
    M, K = Xq.shape
    N = Wq_gate.shape[0]
    if Wq_gate.shape != (N, K) or Wq_up.shape != (N, K):
        raise ValueError("Wq_gate and Wq_up must both be [N, K] with Xq's K")
    if not (Xq.is_contiguous() and Wq_gate.is_contiguous() and Wq_up.is_contiguous()):
        raise ValueError("Xq, Wq_gate and Wq_up must be contiguous")
    _require_like(x_scale, "x_scale", torch.float32, M, Xq)
    _require_like(w_scale_gate, "w_scale_gate", torch.float32, N, Xq)
    _require_like(w_scale_up, "w_scale_up", torch.float32, N, Xq)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=Xq.device)
    _require_out(out, "out", torch.bfloat16, (M, N), Xq)
    st = lib().fp8_linear_swiglu(_ptr(Xq), _ptr(x_scale), _ptr(Wq_gate), _ptr(w_scale_gate), _ptr(Wq_up),
                                 _ptr(w_scale_up), M, N, K, _ptr(out), out.stride(0), _stream(Xq))
    _check(st, "fp8_linear_swiglu")
    return out


def fp8_linear_w8a16_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib().fp8_linear_w8a16_workspace_size(M, N, K))


def fp8_linear_w8a16(X: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
                     out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Weight-only FP8 for small M (<= 64): bf16 activations X [M, K] times the
    dequantized codes Wq [N, K] with per-channel scales w_scale [N], fp32 sums.
    -> Y bf16 [M, N].  `workspace`: a zero-filled uint8 device buffer of at
    least fp8_linear_w8a16_workspace_size bytes (allocated here when None)."""
    _require_cuda(X, "X", torch.bfloat16)
    _require_cuda(Wq, "Wq", torch.uint8)
    M, K = X.shape
    N = Wq.shape[0]
    if Wq.shape != (N, K) or not Wq.is_contiguous():
        raise ValueError("Wq must be a contiguous [N, K] tensor with X's K")
    if X.stride(1) != 1:
        raise ValueError("X rows must be contiguous")
    _require_like(w_scale, "w_scale", torch.float32, N, X)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _require_out(out, "out", torch.bfloat16, (M, N), X)
    wsb = fp8_linear_w8a16_workspace_size(M, N, K) if 0 < M <= 64 else 0
    if workspace is None and wsb:
        workspace = torch.zeros(wsb, dtype=torch.uint8, device=X.device)
    if workspace is not None:   # its size is checked by the library (FP8Q_ERR_INVALID_ARG)
        _require_like(workspace, "workspace", torch.uint8, 0, X)
    st = lib().fp8_linear_w8a16(_ptr(X), X.stride(0), _ptr(Wq), _ptr(w_scale), M, N, K, _ptr(out), out.stride(0),
                                _ptr(workspace) if workspace is not None else None,
                                workspace.numel() if workspace is not None else 0, _stream(X))
    _check(st, "fp8_linear_w8a16")
    return out


def fp8_quant_kv(kv: torch.Tensor, out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None):
    """FP8 KV cache: one amax/448 scale per (token, head) of a K or V tensor.
    kv bf16 [T, H, 128] (head_dim 128, contiguous) -> (codes uint8 [T, H, 128], scales fp32 [T, H]).
    A head's 128 values are one 128-group of the [T, H*128] rows, so this is
    fp8_quant_act in BLOCK128 mode on that view."""
    if kv.dim() != 3 or kv.shape[2] != 128 or not kv.is_contiguous():
        raise ValueError("kv must be a contiguous [tokens, heads, 128] tensor")
    T, H, D = kv.shape
    if out is None:
        q = torch.empty((T, H, D), dtype=torch.uint8, device=kv.device)
        s = torch.empty((T, H), dtype=torch.float32, device=kv.device)
    else:
        q, s = out
    fp8_quant_act(kv.view(T, H * D), BLOCK128, out=(q.view(T, H * D), s.view(T, H)))
    return q, s


def fp8_linear_workspace_size(M: int, N: int, K: int, mode: int = CHANNEL_TOKEN) -> int:
    return int(lib().fp8_linear_workspace_size(M, N, K, int(mode)))


def fp8_linear(Xq: torch.Tensor, x_scale: torch.Tensor, Wq: torch.Tensor, w_scale: torch.Tensor,
               mode: int = CHANNEL_TOKEN, out: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Y bf16 [M, N] = dequant(Xq) . dequant(Wq)^T.  Workspace (small-M path) is
    taken from torch's caching allocator, zero-filled, unless given; a given one
    must have been zero-filled before its first use (every call leaves it all zero)."""
    _require_cuda(Xq, "Xq", torch.uint8)
    _require_cuda(Wq, "Wq", torch.uint8)
    M, K = Xq.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K:
        raise ValueError("Xq and Wq disagree on K")
    if not (Xq.is_contiguous() and Wq.is_contiguous()):
        raise ValueError("Xq and Wq must be contiguous")
    _require_like(x_scale, "x_scale", torch.float32, _numel(scale_shape_act(M, K, mode)), Xq)
    _require_like(w_scale, "w_scale", torch.float32, _numel(scale_shape_weight(N, K, mode)), Xq)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=Xq.device)
    _require_out(out, "out", torch.bfloat16, (M, N), Xq)
    need = fp8_linear_workspace_size(M, N, K, mode)
    if workspace is None and need > 0:
        workspace = torch.zeros(need, dtype=torch.uint8, device=Xq.device)
    if workspace is not None:   # its size is checked by the library (FP8Q_ERR_INVALID_ARG)
        _require_like(workspace, "workspace", torch.uint8, 0, Xq)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().fp8_linear(_ptr(Xq), _ptr(x_scale), _ptr(Wq), _ptr(w_scale), M, N, K, int(mode),
                          _ptr(out), out.stride(0), _ptr(workspace), wbytes, _stream(Xq))
    _check(st, "fp8_linear")
    return out


def device_error(clear: bool = True) -> int:
    """Device-side error word (nonzero after a kernel gave up waiting)."""
    return int(lib().fp8q_device_error(1 if clear else 0))


def version() -> int:
    return int(lib().fp8q_version())


# Short aliases.
quant_weight = fp8_quant_weight
quant_act = fp8_quant_act
linear = fp8_linear
