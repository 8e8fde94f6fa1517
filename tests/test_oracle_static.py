"""Pins of the static-scale quantizer and the percentile calibration.

"Llama 3 精读实录" section 2 calibrates each tensor offline from percentiles of
a calibration set (99.9% and 0.1% quantiles, not min/max) and codes every
element with that fixed scale at run time.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _pins


def test_static_codes_are_the_nearest_values_of_x_over_s():
    x = synth.make_x(16, 512, seed=1)
    for s in (0.01, 0.037, 0.25, 3.0):
        q = oracle.quant_static(x, s)
        quot = (x.float().numpy() / np.float32(s)).astype(np.float32)
        assert np.array_equal(q.ravel(), _pins.encode_argmin(quot.ravel()))


def test_static_scale_one_is_the_plain_e4m3_cast():
    x = (torch.randn(8, 256, generator=torch.Generator().manual_seed(2)) * 30).to(torch.bfloat16)
    q = oracle.quant_static(x, 1.0)
    ref = x.float().clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


def test_static_saturates_outside_the_range():
    x = torch.tensor([[1000.0, -1000.0, 448.0, 0.0] + [1.0] * 12], dtype=torch.bfloat16)
    q = oracle.quant_static(x, 1.0)
    assert q[0, 0] == 0x7E and q[0, 1] == 0xFE and q[0, 2] == 0x7E and q[0, 3] == 0x00


def test_percentile_scale_against_torch_quantile():
    x = synth.make_x(512, 1024, seed=3)          # outlier columns: P99.9 well below the max
    s = oracle.percentile_scale(x)
    xf = x.double().flatten()
    lo, hi = torch.quantile(xf, torch.tensor([0.001, 0.999], dtype=torch.float64)).tolist()
    ref = np.float32(np.float32(max(abs(lo), abs(hi))) / np.float32(448.0))
    assert s == float(ref)
    assert s < float(x.float().abs().max()) / 448.0     # clipped: below the max-based scale


def test_percentile_scale_of_zeros_is_one():
    assert oracle.percentile_scale(torch.zeros(4, 16, dtype=torch.bfloat16)) == 1.0
