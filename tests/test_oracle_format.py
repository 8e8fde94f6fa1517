"""Pins of the oracle's FP8 formats against the pages' printed facts and
against torch's own float8 dtypes (an independent library implementation)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests import _pins

FACTS = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


def test_e4m3_decode_matches_torch_all_256():
    ref = _pins.e4m3_values_torch()
    for c in range(256):
        got = oracle.e4m3_decode(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), hex(c)
        else:
            assert got == ref[c], hex(c)
            assert math.copysign(1, got) == math.copysign(1, ref[c]), hex(c)


def test_e4m3_nan_codes_are_only_7f_ff():
    nans = [c for c in range(256) if math.isnan(oracle.e4m3_decode(c))]
    assert nans == [0x7F, 0xFF]


def test_e4m3_max_finite_is_448_from_page():
    finite = [oracle.e4m3_decode(c) for c in range(256) if not math.isnan(oracle.e4m3_decode(c))]
    assert max(finite) == FACTS["e4m3_max_finite"]["value"] == oracle.e4m3_decode(0x7E)
    assert min(finite) == -448.0 == oracle.e4m3_decode(0xFE)
    assert not any(math.isinf(v) for v in finite)


def test_e5m2_max_finite_is_57344_from_page():
    ref = _pins.e5m2_values_torch()
    got = np.array([oracle.e5m2_decode(c) for c in range(256)])
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))
    fin = got[np.isfinite(got)]
    assert fin.max() == FACTS["e5m2_max_finite"]["value"] == oracle.e5m2_decode(0x7B)


def test_e4m3_every_value_is_integer_multiple_of_2pow_minus9():
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if not math.isnan(v):
            k = v * 512
            assert k == int(k) and abs(k) <= 448 * 512


def test_encode_roundtrip_all_finite_codes_keeps_signed_zero():
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if math.isnan(v):
            continue
        assert oracle.e4m3_encode(v) == c, hex(c)
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(0.0) == 0x00


def test_encode_midpoints_go_to_even_mantissa():
    mags = [oracle.e4m3_decode(c) for c in range(0x7F)]
    for c in range(0x7E):
        mid = (mags[c] + mags[c + 1]) / 2
        assert float(np.float32(mid)) == mid  # exactly representable
        want = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(mid) == want, (hex(c), mid)
        assert oracle.e4m3_encode(-mid) == want | 0x80
        # torch's RNE cast (library) agrees at every midpoint below 464
        t = torch.tensor([mid, -mid], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
        assert t.tolist() == [want, want | 0x80]


def test_encode_saturates_at_448():
    for v in (448.0, 448.0 * (1 + 2 ** -5), 463.99, 464.0, 464.01, 479.0, 480.0, 1e6, 1e30,
              float(np.finfo(np.float32).max)):
        assert oracle.e4m3_encode(v) == 0x7E, v
        assert oracle.e4m3_encode(-v) == 0xFE, v


def test_encode_matches_torch_cast_on_all_bf16_patterns_in_range():
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    f = bits.to(torch.float32)
    keep = torch.isfinite(f) & (f.abs() < 464)
    f = f[keep]
    ref = f.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode_array(f.numpy())
    assert np.array_equal(got, ref)


def test_encode_matches_torch_cast_and_argmin_on_random_floats():
    rng = np.random.default_rng(1234)
    # log-uniform magnitudes from deep subnormal to just below 464, random sign
    mag = np.exp(rng.uniform(np.log(1e-5), np.log(463.9), 200_000)).astype(np.float32)
    v = np.where(rng.random(mag.size) < 0.5, -mag, mag).astype(np.float32)
    got = oracle.e4m3_encode_array(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)
    sub = v[:20_000]
    assert np.array_equal(got[:20_000], _pins.encode_argmin(sub))


def test_encode_argmin_agrees_beyond_torch_range():
    # above 464 torch's cast is not saturating, so the argmin search pins it
    v = np.array([464.0, 470.0, 500.0, 1e4, -1e9, 3.0e38], np.float32)
    assert np.array_equal(oracle.e4m3_encode_array(v), _pins.encode_argmin(v))
