"""The oracle's pins are strong enough to catch plausible mistakes.

Each case plants one mistake in a copy of oracle/fp8_oracle.c (on the CPU,
in a temporary directory), builds it, and runs independent checks against
it: torch's float8 casts, exact rational arithmetic, and the properties the
quantization scheme fixes.  Every mutant must fail at least one check, and
the unmodified source must pass them all.
"""
import ctypes
import os
import re
import subprocess
import tempfile
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth
from tests import _pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "fp8_oracle.c")

MUTANTS = {
    "exponent bias 8": (r"ldexp\(1\.0 \+ m / 8\.0, e - 7\)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "ties away from even": (r"c = \(uint8_t\)\(\(lo & 1\) \? hi : lo\);", "c = (uint8_t)((lo & 1) ? lo : hi);"),
    "no sign on codes": (r"return \(uint8_t\)\(c \| sign\);", "return (uint8_t)c;"),
    "scale amax/447": (r"return num / 448\.0f;", "return num / 447.0f;"),
    "scale by multiplication": (r"volatile float q = x / s;", "volatile float q = x * (1.0f / s);"),
    "min instead of max": (r"if \(a > amax\) amax = a;", "if (a < amax || amax == 0.0f) amax = a;"),
    "w_scale dropped": (r"return \(float\)\(\(double\)xs\[m\] \* \(double\)ws\[n\]", "return (float)((double)xs[m] * 1.0"),
    "operand rows swapped": (r"code_dot\(xq \+ m \* ldx, wq \+ n \* ldw, 0, K\)", "code_dot(xq + n * ldx, wq + m * ldw, 0, K)"),
    "block w_scale row": (r"ws\[\(n / 128\) \* KB \+ kb\]", "ws[(n / 64) * KB + kb]"),
    "block x_scale column": (r"xs\[m \* KB \+ kb\]", "xs[m * KB]"),
    "group of 64": (r"for \(int64_t k = g \* 128; k < g \* 128 \+ 128; \+\+k\) \{", "for (int64_t k = g * 128; k < g * 128 + 64; ++k) {"),
    "amax = 0 gives scale 0": (r"if \(amax == 0\.0f\) return 1\.0f;", "if (amax == 0.0f) return 0.0f;"),
    "rms without the square root": (r"rstd\[r\] = rsqrt_f32_rn\(d\);", "rstd[r] = 1.0f / d;"),
    "rms mean over K - 1": (r"float ms = sq_mean_f32\(acc, K\);", "float ms = sq_mean_f32(acc, K - 1);"),
    "rms sum of |x| not x^2": (r"uint64_t sq = m \* m;", "uint64_t sq = m;"),
    "rms subnormal exponent": (r"if \(e != 0\) \{ m \+= 128; p = e - 1; \}", "if (e != 0) { m += 128; p = e; }"),
    "rsqrt rounds up": (r"uint64_t Mid = A \+ B;", "uint64_t Mid = A + A;"),
    "rms eps ignored": (r"volatile float d = ms \+ eps;", "volatile float d = ms;"),
    "rms gamma dropped": (r"volatile float g = bf16_to_float\(gamma\[k\]\) \* bf16_to_float\(h\);",
                          "volatile float g = bf16_to_float(h);"),
    "swiglu without the sigmoid": (r"float_to_bf16\(\(float\)\(gb / \(1\.0 \+ exp\(-gb\)\)\)\)",
                                   "float_to_bf16((float)gb)"),
    "swiglu sigmoid sign": (r"exp\(-gb\)", "exp(gb)"),
    "swiglu up dropped": (r"volatile float p = bf16_to_float\(sb\) \* \(float\)ub;",
                          "volatile float p = bf16_to_float(sb);"),
    "bf16 scale not rounded": (r"float r = bf16_to_float\(float_to_bf16\(s\)\);", "float r = s;"),
    "w8a16 w_scale dropped": (r"y\[m \* N \+ n\] = \(float\)\(acc \* \(double\)ws\[n\]\);",
                              "y[m * N + n] = (float)acc;"),
    "w8a16 weight transposed": (r"orc_e4m3_decode\(wq\[n \* K \+ k\]\)", "orc_e4m3_decode(wq[k * N + n])"),
    "static scale ignored": (r"q\[r \* ldq \+ k\] = code_of\(bf16_to_float\(x\[r \* ld \+ k\]\), s\);",
                             "q[r * ldq + k] = code_of(bf16_to_float(x[r * ld + k]), 1.0f);"),
}


def build_variant(src_text, tmp):
    c = os.path.join(tmp, "o.c")
    so = os.path.join(tmp, "o.so")
    open(c, "w").write(src_text)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
                           "-Wno-unused-variable", c, "-o", so, "-lm"])
    L = ctypes.CDLL(so)
    P, I = ctypes.c_void_p, ctypes.c_int64
    L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.orc_e4m3_decode.restype = ctypes.c_double
    L.orc_e4m3_encode_n.argtypes = [P, I, P]
    for f in ("orc_quant_rows", "orc_quant_groups128", "orc_quant_blocks128", "orc_quant_rows_s16"):
        getattr(L, f).argtypes = [P, I, I, I, P, I, P]
    L.orc_linear.argtypes = [P, P, P, P, I, I, I, I, I, ctypes.c_int, P]
    L.orc_rmsnorm_rstd.argtypes = [P, I, I, I, ctypes.c_float, P]
    L.orc_rmsnorm_quant_rows.argtypes = [P, P, I, I, I, ctypes.c_float, ctypes.c_int, P, I, P, P, P]
    L.orc_linear_swiglu.argtypes = [P, P, P, P, P, P, I, I, I, P]
    L.orc_quant_static.argtypes = [P, I, I, I, ctypes.c_float, P, I]
    L.orc_linear_w8a16.argtypes = [P, P, P, I, I, I, P]
    return L


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def checks(L):
    """Returns the names of the independent checks this build fails."""
    failed = []
    vals = _pins.e4m3_values_torch()
    dec = np.array([L.orc_e4m3_decode(c) for c in range(256)])
    if not np.all((np.isnan(dec) & np.isnan(vals)) | (dec == vals)):
        failed.append("decode vs torch")
    # encoder vs torch RNE cast on every bf16 pattern below 464
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()
    f = bits[torch.isfinite(bits) & (bits.abs() < 464)].numpy().astype(np.float32)
    out = np.empty(f.size, np.uint8)
    L.orc_e4m3_encode_n(_p(f), f.size, _p(out))
    if not np.array_equal(out, torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()):
        failed.append("encode vs torch")
    # row quantization: max element -> +-448 code, scale ~ amax/448, codes ~ x/s
    x = synth.make_x(8, 256, seed=3)
    xb = x.view(torch.int16).numpy().view(np.uint16).copy()
    q = np.empty((8, 256), np.uint8)
    s = np.empty(8, np.float32)
    L.orc_quant_rows(_p(xb), 8, 256, 256, _p(q), 256, _p(s))
    xf = x.float().numpy().astype(np.float64)
    for r in range(8):
        i = np.abs(xf[r]).argmax()
        amax = np.abs(xf[r]).max()
        if (q[r, i] & 0x7F) != 0x7E or abs(float(s[r]) * 448 - amax) > amax * 2 ** -22:
            failed.append("row amax -> 448")
            break
    quot = (x.float().numpy() / s[:, None]).astype(np.float32)
    if not np.array_equal(q.ravel(), _pins.encode_argmin(quot.ravel())):
        failed.append("row codes vs argmin of x/s")
    # IEEE division (not x * (1/s)): every bf16 x <= 1632 against amax 1632
    allv = torch.arange(0, 0x7F80, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    xs_ = allv[(allv.float() <= 1632.0) & (allv.float() >= 0.05)][:1023]   # includes 0.0747, 0.1494
    row = torch.cat([torch.tensor([1632.0], dtype=torch.bfloat16), xs_]).reshape(1, -1)
    rb = row.view(torch.int16).numpy().view(np.uint16).copy()
    qd = np.empty(rb.shape, np.uint8)
    sd = np.empty(1, np.float32)
    L.orc_quant_rows(_p(rb), 1, rb.shape[1], rb.shape[1], _p(qd), rb.shape[1], _p(sd))
    sref = np.float32(np.float32(1632.0) / np.float32(448.0))
    want = torch.from_numpy((row.float().numpy() / sref).astype(np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()
    if not np.array_equal(qd, want):
        failed.append("IEEE division")
    # scales rounded to bf16 before the codes: the rounded fp32 scales, codes by argmin
    q16 = np.empty((8, 256), np.uint8)
    s16 = np.empty(8, np.float32)
    L.orc_quant_rows_s16(_p(xb), 8, 256, 256, _p(q16), 256, _p(s16))
    if not np.array_equal(s16, torch.from_numpy(s.copy()).to(torch.bfloat16).float().numpy()) or \
            not np.array_equal(q16.ravel(), _pins.encode_argmin((x.float().numpy() / s16[:, None]).astype(np.float32).ravel())):
        failed.append("bf16 scales")
    # static scale: codes of x / s for a fixed s
    qs_ = np.empty((8, 256), np.uint8)
    L.orc_quant_static(_p(xb), 8, 256, 256, ctypes.c_float(0.05), _p(qs_), 256)
    if not np.array_equal(qs_.ravel(), _pins.encode_argmin((x.float().numpy() / np.float32(0.05)).astype(np.float32).ravel())):
        failed.append("static scale")
    z = np.zeros((2, 256), np.uint16)
    qz = np.empty((2, 256), np.uint8)
    sz = np.empty(2, np.float32)
    L.orc_quant_rows(_p(z), 2, 256, 256, _p(qz), 256, _p(sz))
    if not (np.all(sz == 1.0) and np.all(qz == 0)):
        failed.append("zero rows")
    # groups: each group equals a row quantization of that group alone
    xg = synth.make_x(3, 384, seed=4)
    xgb = xg.view(torch.int16).numpy().view(np.uint16).copy()
    qg = np.empty((3, 384), np.uint8)
    sg = np.empty((3, 3), np.float32)
    L.orc_quant_groups128(_p(xgb), 3, 384, 384, _p(qg), 384, _p(sg))
    for g in range(3):
        sub = np.ascontiguousarray(xgb[:, g * 128:(g + 1) * 128])
        qs = np.empty((3, 128), np.uint8)
        ss = np.empty(3, np.float32)
        L.orc_quant_rows(_p(sub), 3, 128, 128, _p(qs), 128, _p(ss))
        amax = np.abs(xg.float().numpy()[:, g * 128:(g + 1) * 128]).max(axis=1)
        if not (np.array_equal(qs, qg[:, g * 128:(g + 1) * 128]) and np.array_equal(ss, sg[:, g])) or \
                np.any(np.abs(sg[:, g].astype(np.float64) * 448 - amax) > amax * 2 ** -22):
            failed.append("groups")
            break
    # linear vs exact rationals, both modes, non-square
    rng = np.random.default_rng(5)
    M, N, K = 3, 130, 256
    xq = rng.integers(0, 256, (M, K)).astype(np.uint8)
    wq = rng.integers(0, 256, (N, K)).astype(np.uint8)
    xq[(xq & 0x7F) == 0x7F] = 0x38
    wq[(wq & 0x7F) == 0x7F] = 0x38
    xs = rng.uniform(0.1, 2, M).astype(np.float32)
    ws = rng.uniform(0.01, 0.1, N).astype(np.float32)
    y = np.empty((M, N), np.float32)
    L.orc_linear(_p(xq), _p(xs), _p(wq), _p(ws), M, N, K, K, K, 0, _p(y))
    for m, n in [(0, 0), (2, 129), (1, 64)]:
        e = sum(Fraction(float(vals[a])) * Fraction(float(vals[b])) for a, b in zip(xq[m], wq[n]))
        e = float(e * Fraction(float(xs[m])) * Fraction(float(ws[n])))
        if abs(float(y[m, n]) - e) > _pins.f32_ulp(e):
            failed.append("linear channel vs rationals")
            break
    xsb = rng.uniform(0.1, 2, (M, K // 128)).astype(np.float32)
    wsb = rng.uniform(0.01, 0.1, ((N + 127) // 128, K // 128)).astype(np.float32)
    L.orc_linear(_p(xq), _p(xsb), _p(wq), _p(wsb), M, N, K, K, K, 1, _p(y))
    for m, n in [(0, 0), (2, 129), (1, 64)]:
        e = Fraction(0)
        for k in range(K):
            e += Fraction(float(vals[xq[m, k]])) * Fraction(float(vals[wq[n, k]])) * \
                Fraction(float(xsb[m, k // 128])) * Fraction(float(wsb[n // 128, k // 128]))
        if abs(float(y[m, n]) - float(e)) > _pins.f32_ulp(float(e)) * 2:
            failed.append("linear block vs rationals")
            break
    # RMSNorm: rstd against the float64 mean of squares (1 ulp), normalised
    # rows against torch's float64 rms_norm (two bf16 roundings)
    Kr = 512
    xr = synth.make_x(4, Kr, seed=6)
    xrb = xr.view(torch.int16).numpy().view(np.uint16).copy()
    gr = (1.0 + 0.1 * torch.randn(Kr, generator=torch.Generator().manual_seed(6))).to(torch.bfloat16)
    grb = gr.view(torch.int16).numpy().view(np.uint16).copy()
    rs = np.empty(4, np.float32)
    L.orc_rmsnorm_rstd(_p(xrb), 4, Kr, Kr, ctypes.c_float(1e-5), _p(rs))
    ms = (xr.double() ** 2).mean(dim=1).float()
    rref = (1.0 / torch.sqrt((ms + torch.tensor(1e-5, dtype=torch.float32)).double())).float().numpy()
    if np.abs(rs.view(np.int32).astype(np.int64) - rref.view(np.int32).astype(np.int64)).max() > 1:
        failed.append("rmsnorm rstd")
    # rstd exactly: rational mean of squares, mpmath reciprocal square root
    if any(rs[i] != _pins.rmsnorm_rstd_exact(xrb[i], 1e-5) for i in range(4)):
        failed.append("rmsnorm rstd exact")
    xe = synth.make_x(24, 64, seed=8)
    xeb = xe.view(torch.int16).numpy().view(np.uint16).copy()
    re_ = np.empty(24, np.float32)
    L.orc_rmsnorm_rstd(_p(xeb), 24, 64, 64, ctypes.c_float(1e-5), _p(re_))
    if any(re_[i] != _pins.rmsnorm_rstd_exact(xeb[i], 1e-5) for i in range(24)):
        failed.append("rmsnorm rstd exact, short rows")
    xt = np.zeros((1, 64), np.uint16)
    xt[0, 5] = 0x0001                       # the smallest subnormal, with a normal value beside it
    xt[0, 6] = 0x3F80                       # 1.0
    rt = np.empty(1, np.float32)
    L.orc_rmsnorm_rstd(_p(xt), 1, 64, 64, ctypes.c_float(0.0), _p(rt))
    if rt[0] != _pins.rmsnorm_rstd_exact(xt[0], 0.0):
        failed.append("rmsnorm rstd subnormal")
    qr = np.empty((4, Kr), np.uint8)
    sr = np.empty(4, np.float32)
    yr = np.empty((4, Kr), np.uint16)
    ro = np.empty(4, np.float32)
    L.orc_rmsnorm_quant_rows(_p(xrb), _p(grb), 4, Kr, Kr, ctypes.c_float(1e-5), 0, _p(qr), Kr, _p(sr), _p(yr),
                             _p(ro))
    yref = torch.nn.functional.rms_norm(xr.double(), (Kr,), weight=gr.double(), eps=1e-5)
    yt = torch.from_numpy(yr.astype(np.int16)).view(torch.bfloat16).double()
    if not torch.all((yt - yref).abs() <= 2.0 ** -7 * yref.abs() * 1.001 + 1e-30):
        failed.append("rmsnorm rows")
    # SwiGLU: bf16(bf16(silu(g)) * u) against torch's float64 silu on the
    # (separately checked) linear outputs rounded to bf16 by torch
    wu = rng.integers(0, 256, (N, K)).astype(np.uint8)
    wu[(wu & 0x7F) == 0x7F] = 0x38
    wsu = rng.uniform(0.01, 0.1, N).astype(np.float32)
    act = np.empty((M, N), np.uint16)
    L.orc_linear_swiglu(_p(xq), _p(xs), _p(wq), _p(ws), _p(wu), _p(wsu), M, N, K, _p(act))
    gE = np.empty((M, N), np.float32)
    uE = np.empty((M, N), np.float32)
    L.orc_linear(_p(xq), _p(xs), _p(wq), _p(ws), M, N, K, K, K, 0, _p(gE))
    L.orc_linear(_p(xq), _p(xs), _p(wu), _p(wsu), M, N, K, K, K, 0, _p(uE))
    gb = torch.from_numpy(gE).to(torch.bfloat16)
    ub = torch.from_numpy(uE).to(torch.bfloat16)
    aref = (torch.nn.functional.silu(gb.double()).to(torch.bfloat16) * ub).view(torch.int16).numpy().view(np.uint16)
    if not np.array_equal(act, aref):
        failed.append("swiglu")
    # weight-only FP8: bf16 activations times dequantized codes, vs rationals
    xw = synth.make_x(2, K, seed=7)
    xwb = xw.view(torch.int16).numpy().view(np.uint16).copy()
    yw = np.empty((2, N), np.float32)
    L.orc_linear_w8a16(_p(xwb), _p(wq), _p(ws), 2, N, K, _p(yw))
    xwf = xw.float().numpy()
    for m, n in [(0, 0), (1, 129), (1, 64)]:
        e = sum(Fraction(float(a)) * Fraction(float(vals[b])) for a, b in zip(xwf[m], wq[n]))
        e = float(e * Fraction(float(ws[n])))
        if abs(float(yw[m, n]) - e) > _pins.f32_ulp(e):
            failed.append("w8a16 vs rationals")
            break
    return failed


def test_unmodified_oracle_passes_every_check():
    with tempfile.TemporaryDirectory() as tmp:
        assert checks(build_variant(open(SRC).read(), tmp)) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    pat, rep = MUTANTS[name]
    src = open(SRC).read()
    mutated, n = re.subn(pat, rep, src)
    assert n >= 1, f"mutation '{name}' did not apply"
    with tempfile.TemporaryDirectory() as tmp:
        failed = checks(build_variant(mutated, tmp))
    assert failed, f"planted mistake '{name}' passed every check"
