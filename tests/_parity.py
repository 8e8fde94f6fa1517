"""Shared helpers of the GPU parity tests (tests only)."""
from __future__ import annotations

import numpy as np
import torch

import oracle


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (8 significant bits)."""
    a = np.abs(v.astype(np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -133)))
    return 2.0 ** (e - 7)


def y_tolerance(y_ref: np.ndarray, scale_max: float) -> np.ndarray:
    """Output tolerance: 4e-3 * max|y_ref| over the whole output, plus one bf16
    ulp of each element.  The first term bounds fp32 accumulation-order and
    scale-product rounding differences against the exact oracle; the second
    is the final rounding to bf16."""
    return 4e-3 * scale_max + bf16_ulp(y_ref)


def assert_y_close(y_gpu: np.ndarray, y_ref: np.ndarray, scale_max: float | None = None, what=""):
    y_gpu = y_gpu.astype(np.float64)
    y_ref = y_ref.astype(np.float64)
    if scale_max is None:
        scale_max = float(np.abs(y_ref).max()) if y_ref.size else 0.0
    err = np.abs(y_gpu - y_ref)
    tol = y_tolerance(y_ref, scale_max)
    bad = err > tol
    if bad.any():
        i = np.argmax(err - tol)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outputs out of tolerance; worst at flat "
                             f"index {i}: gpu {y_gpu.flat[i]} ref {y_ref.flat[i]} tol {tol.flat[i]}")


def codes_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def assert_codes_equal(gpu: torch.Tensor, ref: np.ndarray, what=""):
    g = codes_np(gpu)
    if not np.array_equal(g, ref):
        d = np.argwhere(g != ref)
        i = tuple(d[0])
        raise AssertionError(f"{what}: {len(d)} codes differ; first at {i}: gpu {g[i]:#04x} ref {ref[i]:#04x}")


def assert_scales_equal(gpu: torch.Tensor, ref: np.ndarray, what=""):
    g = gpu.detach().cpu().numpy()
    if not np.array_equal(g.view(np.uint32), ref.astype(np.float32).view(np.uint32)):
        d = np.argwhere(g != ref)
        raise AssertionError(f"{what}: {len(d)} scales differ; first at {tuple(d[0])}")


def oracle_rows_for(x_cpu: torch.Tensor, rows: np.ndarray, mode: int):
    """Oracle activation codes and scales of the selected rows only (a row's
    quantization does not depend on the other rows)."""
    sub = x_cpu[torch.as_tensor(rows)].contiguous()
    return oracle.quant_act(sub, mode)


def oracle_weight_rows_for(w_cpu: torch.Tensor, rows: np.ndarray, mode: int):
    """Oracle codes/scales for selected weight rows.  In block mode the whole
    128-row blocks holding them are quantized (the block amax spans them)."""
    if mode == oracle.CHANNEL_TOKEN:
        sub = w_cpu[torch.as_tensor(rows)].contiguous()
        q, s = oracle.quant_rows(sub)
        return q, s, {int(r): i for i, r in enumerate(rows)}
    blocks = sorted({int(r) // 128 for r in rows})
    qs, ss, index = [], [], {}
    for j, b in enumerate(blocks):
        blk = w_cpu[b * 128:(b + 1) * 128].contiguous()
        q, s = oracle.quant_blocks128(blk)
        qs.append(q)
        ss.append(s)
    for r in rows:
        j = blocks.index(int(r) // 128)
        index[int(r)] = (j, int(r) % 128)
    return qs, ss, index
