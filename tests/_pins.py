"""Independent cross-checks used to pin the oracle (test helpers only).

Nothing here is shared with the oracle or with the GPU library.  The E4M3
value set is taken from torch's own float8_e4m3fn dtype (a library routine),
and the encoder is a vectorised argmin over all candidate values, written
differently from the oracle's bisection.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import torch


def e4m3_values_torch() -> np.ndarray:
    """float64 value of each of the 256 codes, via torch's float8_e4m3fn cast."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def e5m2_values_torch() -> np.ndarray:
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e5m2).to(torch.float64).numpy()


_VALS = None


def _finite_table():
    global _VALS
    if _VALS is None:
        v = e4m3_values_torch()
        codes = np.array([c for c in range(256) if np.isfinite(v[c])], np.int64)
        _VALS = (codes, v[codes])
    return _VALS


def encode_argmin(x: np.ndarray) -> np.ndarray:
    """Nearest finite E4M3 code to each float32 in x; exact ties go to the
    code with an even mantissa; the sign bit follows the sign of x (so -0 and
    negative values that round to zero give 0x80)."""
    codes, vals = _finite_table()
    x = np.asarray(x, np.float32).astype(np.float64).ravel()
    out = np.empty(x.size, np.uint8)
    for lo in range(0, x.size, 4096):
        xs = x[lo:lo + 4096]
        neg = np.signbit(xs)
        # beyond 896 the nearest value is 448 whatever the magnitude; clipping
        # keeps the float64 distances resolvable for huge inputs
        mag = np.minimum(np.abs(xs), 896.0)
        pos = codes < 128
        pc, pv = codes[pos], vals[pos]
        d = np.abs(mag[:, None] - pv[None, :])
        best = d.min(axis=1, keepdims=True)
        cand = d == best
        # among equal distances prefer the even code (mantissa LSB 0)
        score = np.where(cand, np.where(pc[None, :] % 2 == 0, 2, 1), 0)
        idx = score.argmax(axis=1)
        c = pc[idx].astype(np.uint8)
        out[lo:lo + 4096] = np.where(neg, c | 0x80, c)
    return out


def exact_linear_channel(xq, xs, wq, ws) -> list:
    """Exact rational Y[m][n] = sum_k (E4M3(xq)*xs[m]) * (E4M3(wq)*ws[n])."""
    vals = e4m3_values_torch()
    fx = [[Fraction(float(vals[c])) for c in row] for row in xq]
    fw = [[Fraction(float(vals[c])) for c in row] for row in wq]
    M, N = len(fx), len(fw)
    out = []
    for m in range(M):
        row = []
        for n in range(N):
            acc = Fraction(0)
            for a, b in zip(fx[m], fw[n]):
                acc += (a * Fraction(float(xs[m]))) * (b * Fraction(float(ws[n])))
            row.append(acc)
        out.append(row)
    return out


def exact_linear_block(xq, xs, wq, ws) -> list:
    """Exact rational block-mode output: scales picked per 128-wide K slice."""
    vals = e4m3_values_torch()
    M, K = len(xq), len(xq[0])
    N = len(wq)
    out = []
    for m in range(M):
        row = []
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                kb = k // 128
                a = Fraction(float(vals[xq[m][k]])) * Fraction(float(xs[m][kb]))
                b = Fraction(float(vals[wq[n][k]])) * Fraction(float(ws[n // 128][kb]))
                acc += a * b
            row.append(acc)
        out.append(row)
    return out


def f32_ulp(v: float) -> float:
    v = abs(np.float32(v))
    return float(np.spacing(np.float32(v))) if v > 0 else float(np.spacing(np.float32(0)))


def f32_nearest(v: Fraction) -> np.float32:
    """The fp32 nearest to the exact rational v (ties to even).  Python's
    Fraction -> float is correctly rounded to double; rounding that double to
    fp32 again is wrong only when it lands exactly on an fp32 midpoint while v
    does not, which is then settled by comparing v with that midpoint."""
    d = float(v)
    f = np.float32(d)
    if Fraction(d) != v:
        lo = np.nextafter(f, np.float32(-np.inf), dtype=np.float32)
        hi = np.nextafter(f, np.float32(np.inf), dtype=np.float32)
        for a, b in ((lo, f), (f, hi)):
            mid = (Fraction(float(a)) + Fraction(float(b))) / 2
            if Fraction(d) == mid:
                return b if v > mid else a
    return f


def bf16_bits_sum_of_squares(bits: np.ndarray) -> Fraction:
    """Exact sum of x^2 over bf16 bit patterns, in Python integers: each bf16
    value is an integer multiple of 2^-133."""
    total = 0
    for b in np.asarray(bits, np.uint16).ravel().tolist():
        e, m = (b >> 7) & 0xFF, b & 0x7F
        k = m if e == 0 else (128 + m) << (e - 1)    # |x| = k * 2^-133
        total += k * k
    return Fraction(total, 2 ** 266)


def rsqrt_f32_mpmath(d: np.float32) -> np.float32:
    """1 / sqrt(d) rounded to fp32 through mpmath at 200 bits (then to double,
    then fp32; 1/sqrt of an fp32 value is never an fp32 midpoint, and a
    200-bit value that rounds to a double midpoint of fp32 is asserted absent)."""
    import mpmath
    with mpmath.workprec(200):
        v = 1 / mpmath.sqrt(mpmath.mpf(float(d)))
        dv = float(v)
    f = np.float32(dv)
    lo = np.nextafter(f, np.float32(0), dtype=np.float32)
    hi = np.nextafter(f, np.float32(np.inf), dtype=np.float32)
    for a, b in ((lo, f), (f, hi)):
        assert Fraction(dv) != (Fraction(float(a)) + Fraction(float(b))) / 2, "double landed on an fp32 midpoint"
    return f


def rmsnorm_rstd_exact(bits_row: np.ndarray, eps: float) -> np.float32:
    """rstd = RN32(1 / sqrt(RN32(RN32(mean x^2) + eps))) from exact arithmetic."""
    K = np.asarray(bits_row).size
    ms = f32_nearest(bf16_bits_sum_of_squares(bits_row) / K)
    d = np.float32(ms + np.float32(eps))       # one fp32 addition
    return rsqrt_f32_mpmath(d)
