"""Pins of the oracle's quantizers: properties that the scheme on the pages
fixes (symmetric amax/448 scale per unit, E4M3 codes), checked without
re-typing the oracle's formulas.

Scheme: Llama-3.1-8B-Instruct-FP8-Dynamic explainer, FP8 动态量化 table
(per-output-channel minmax weights, dynamic per-token activations);
Llama-3.2-3B-Instruct-FP8-Block explainer, quantization_config table
(128x128 weight blocks, dynamic groups of 128 for activations).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _pins

VALS = _pins.e4m3_values_torch()


def _f(xbf16):
    return xbf16.to(torch.float32).numpy().astype(np.float64)


def _check_unit(x, q, s):
    """x: float64 values of one unit, q: its codes, s: its scale."""
    amax = np.abs(x).max()
    if amax == 0:
        assert s == 1.0 and np.all((q & 0x7F) == 0)
        return
    # the unit's largest |x| lands on the largest code, +-448
    i = np.abs(x).argmax()
    assert (q[i] & 0x7F) == 0x7E
    assert (q[i] & 0x80) == (0x80 if x[i] < 0 else 0)
    # s is amax/448 up to one fp32 rounding
    assert abs(float(s) * 448 - amax) <= amax * 2.0 ** -23
    # every code decodes to within half an E4M3 step of x/s
    d = VALS[q] * float(s)
    err = np.abs(d - x)
    # step of the E4M3 binade containing |x|/s (subnormal step 2^-9)
    r = np.abs(x) / float(s)
    e = np.floor(np.log2(np.maximum(r, 2.0 ** -6)))
    step = 2.0 ** (e - 3)
    assert np.all(err <= (0.5 * step + 2.0 ** -20 * r) * float(s) + 1e-30)
    # signs kept (zero codes may be +-0)
    nz = (q & 0x7F) != 0
    assert np.all(np.signbit(VALS[q][nz]) == np.signbit(x[nz]))


def test_rows_unit_properties():
    x = synth.make_x(37, 384, seed=3)
    q, s = oracle.quant_rows(x)
    xf = _f(x)
    assert q.shape == (37, 384) and s.shape == (37,)
    for r in range(37):
        _check_unit(xf[r], q[r], s[r])


def test_groups128_unit_properties_and_shapes():
    x = synth.make_x(9, 512, seed=4)
    q, s = oracle.quant_groups128(x)
    assert s.shape == (9, 4)
    xf = _f(x)
    for m in range(9):
        for g in range(4):
            _check_unit(xf[m, g * 128:(g + 1) * 128], q[m, g * 128:(g + 1) * 128], s[m, g])


def test_blocks128_unit_properties_and_ragged_rows():
    w = synth.make_w(300, 256, seed=5)   # 3 row-tiles, the last has 44 rows
    q, s = oracle.quant_blocks128(w)
    assert s.shape == (3, 2)
    wf = _f(w)
    for nb in range(3):
        for kb in range(2):
            blk = wf[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            qb = q[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            _check_unit(blk.ravel(), qb.ravel(), s[nb, kb])


def test_zero_unit_gets_unit_scale_and_zero_codes():
    x = torch.zeros(3, 256, dtype=torch.bfloat16)
    x[1, 5] = -2.5
    q, s = oracle.quant_rows(x)
    assert s[0] == 1.0 and s[2] == 1.0 and np.all(q[0] == 0) and np.all(q[2] == 0)
    assert q[1, 5] == 0xFE and s[1] == np.float32(2.5) / np.float32(448)
    qg, sg = oracle.quant_groups128(x)
    assert sg[1, 0] == s[1] and sg[1, 1] == 1.0


def test_negation_flips_only_sign_bits():
    x = synth.make_x(8, 256, seed=6)
    q1, s1 = oracle.quant_rows(x)
    q2, s2 = oracle.quant_rows(-x)
    assert np.array_equal(s1, s2)
    assert np.array_equal(q1 ^ 0x80, q2)


def test_power_of_two_rescaling_is_exact():
    # bf16 * 2^k is exact, so scales scale by 2^k and codes do not change
    x = synth.make_x(8, 256, seed=7)
    q1, s1 = oracle.quant_rows(x)
    for k in (-12, -3, 5):
        q2, s2 = oracle.quant_rows(x * 2.0 ** k)
        assert np.array_equal(q1, q2)
        assert np.array_equal(s2, (s1.astype(np.float64) * 2.0 ** k).astype(np.float32))


def test_monotone_within_a_row():
    x = torch.linspace(-50, 50, 2048).to(torch.bfloat16).reshape(1, -1)
    q, s = oracle.quant_rows(x)
    d = VALS[q[0]]
    assert np.all(np.diff(d) >= 0)


def test_groups_with_k128_reduce_to_rows():
    x = synth.make_x(11, 128, seed=8)
    qg, sg = oracle.quant_groups128(x)
    qr, sr = oracle.quant_rows(x)
    assert np.array_equal(qg, qr) and np.array_equal(sg[:, 0], sr)


def test_single_block_reduces_to_one_row_of_16384():
    w = synth.make_w(128, 128, seed=9)
    qb, sb = oracle.quant_blocks128(w)
    qr, sr = oracle.quant_rows(w.reshape(1, 128 * 128))
    assert np.array_equal(qb.ravel(), qr.ravel()) and sb[0, 0] == sr[0]


def test_blocks_are_independent_of_their_neighbours():
    w = synth.make_w(256, 384, seed=10)
    q, s = oracle.quant_blocks128(w)
    for nb in range(2):
        for kb in range(3):
            t = w[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128].contiguous()
            qt, st = oracle.quant_blocks128(t)
            assert st[0, 0] == s[nb, kb]
            assert np.array_equal(qt, q[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128])


def test_groups_are_independent_of_their_neighbours():
    x = synth.make_x(4, 384, seed=11)
    q, s = oracle.quant_groups128(x)
    for g in range(3):
        qt, st = oracle.quant_rows(x[:, g * 128:(g + 1) * 128].contiguous())
        assert np.array_equal(st, s[:, g]) and np.array_equal(qt, q[:, g * 128:(g + 1) * 128])


def test_weight_channel_quant_is_the_row_quant():
    w = synth.make_w(64, 256, seed=12)
    a = oracle.quant_weight(w, oracle.CHANNEL_TOKEN)
    b = oracle.quant_act(w, oracle.CHANNEL_TOKEN)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_codes_match_independent_encoder_on_synthetic_rows():
    x = synth.make_x(16, 256, seed=0, n_out=2)
    q, s = oracle.quant_rows(x)
    xf = x.to(torch.float32).numpy()
    quot = (xf / s[:, None]).astype(np.float32)   # numpy fp32 IEEE division
    assert np.array_equal(q.ravel(), _pins.encode_argmin(quot.ravel()))


def _division_rows(amax):
    """Rows whose amax is `amax`, holding every bf16 value in [0, amax]."""
    allv = torch.arange(0, 0x7F80, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    xs = allv[allv.float() <= amax]
    per = 1023
    rows = []
    for i in range(0, xs.numel(), per):
        chunk = xs[i:i + per]
        row = torch.zeros(per + 1, dtype=torch.bfloat16)
        row[0] = amax
        row[1:1 + chunk.numel()] = chunk
        rows.append(row)
    return torch.stack(rows)


@pytest.mark.parametrize("amax", [1632.0, 191.0, 66.0, 8224768.0])
def test_codes_follow_ieee_division(amax):
    """Reading R3: the code is E4M3 of the IEEE fp32 quotient x / s.  For these
    amax values some x give a different code under x * (1/s); numpy's fp32
    division and torch's fp8 cast fix the expected codes independently."""
    x = _division_rows(amax)
    q, s = oracle.quant_rows(x)
    s_ref = np.float32(np.float32(amax) / np.float32(448.0))
    assert np.all(s == s_ref)
    xf = x.float().numpy()
    want = torch.from_numpy((xf / s_ref).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    recip = torch.from_numpy((xf * np.float32(np.float32(1) / s_ref)).astype(np.float32)) \
        .to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.any(want != recip)          # the case really separates the two readings
    assert np.array_equal(q, want)


# ------------------------------------------------- scales rounded to bf16
# The FP8 checkpoints store bf16 scales (the 70B byte count pins it, see
# test_policy.py); with scale_bf16 the scale is rounded to bf16 before the
# codes are computed, so the codes are those of a bf16-scale checkpoint.

def _bf16_round(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("kind", ["rows", "groups", "blocks"])
def test_bf16_scales_are_the_rounded_fp32_scales(kind):
    x = synth.make_x(300, 512, seed=21)
    f = {"rows": oracle.quant_rows, "groups": oracle.quant_groups128, "blocks": oracle.quant_blocks128}[kind]
    _, s32 = f(x)
    q16, s16 = f(x, scale_bf16=True)
    assert np.array_equal(s16, _bf16_round(s32))
    # codes: the nearest E4M3 value of fl32(x / s16), by the independent argmin encoder
    xf = x.float().numpy()
    if kind == "rows":
        sx = np.repeat(s16[:, None], 512, axis=1)
    elif kind == "groups":
        sx = np.repeat(s16, 128, axis=1)
    else:
        sx = np.repeat(np.repeat(s16, 128, axis=0)[:300], 128, axis=1)
    quot = (xf / sx).astype(np.float32)
    assert np.array_equal(q16.ravel(), _pins.encode_argmin(quot.ravel()))


def test_bf16_scale_rounding_down_saturates_the_max_element():
    # amax = 1632: 1632/448 = 3.642857 rounds to bf16 3.640625 (down), so
    # amax / s = 448.28 > 448 and the max element saturates to 0x7E
    x = torch.zeros(1, 16, dtype=torch.bfloat16)
    x[0, 0] = 1632.0
    x[0, 1] = -1632.0
    q, s = oracle.quant_rows(x, scale_bf16=True)
    assert s[0] == np.float32(3.640625)
    assert q[0, 0] == 0x7E and q[0, 1] == 0xFE


def test_bf16_scale_of_zero_and_tiny_units_is_one():
    x = torch.zeros(2, 16, dtype=torch.bfloat16)
    x[1, 3] = 2.0 ** -133                        # amax/448 rounds to zero in bf16
    q, s = oracle.quant_rows(x, scale_bf16=True)
    assert np.all(s == 1.0) and np.all(q == 0)
