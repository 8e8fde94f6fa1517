"""GPU quantize kernels vs the oracle: codes and scales bit-exact.

Per-token / per-channel (one amax/448 scale per row), per-128-group and
per-128x128-block schemes of the FP8-Dynamic and FP8-Block checkpoints.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import fp8_w8a8_quantized_amax_b200 as fq
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from fp8_w8a8_quantized_amax_b200 import build
    build.build()
    fq.device_error(clear=True)
    yield
    assert fq.device_error(clear=True) == 0


@pytest.mark.parametrize("M,K", [(1, 16), (3, 48), (17, 256), (129, 384), (64, 3072), (5, 4096),
                                 (2051, 3072), (1000, 1040), (301, 4096),
                                 (2, 14336), (3, 28672), (2, 65536 + 16), (1, 131072)])
def test_rows_bit_exact(M, K):
    x = synth.make_x(M, K, seed=M + K)
    q, s = fq.fp8_quant_act(x.to(DEV), fq.CHANNEL_TOKEN)
    rq, rs = oracle.quant_rows(x)
    P.assert_codes_equal(q, rq, f"rows {M}x{K}")
    P.assert_scales_equal(s, rs, f"rows {M}x{K}")


@pytest.mark.parametrize("M,K", [(1, 128), (5, 384), (33, 3072), (300, 256),
                                 (4100, 3072),    # 98,400 groups: 6 per half warp, one pass on 148 SMs
                                 (5000, 3072),    # 120,000 groups: 8 per half warp, one pass
                                 (9000, 3072)])   # 216,000 groups: 8 per half warp, a second pass
def test_groups_bit_exact(M, K):
    x = synth.make_x(M, K, seed=7 * M + K)
    q, s = fq.fp8_quant_act(x.to(DEV), fq.BLOCK128)
    rq, rs = oracle.quant_groups128(x)
    assert tuple(s.shape) == (M, K // 128)
    P.assert_codes_equal(q, rq, f"groups {M}x{K}")
    P.assert_scales_equal(s, rs, f"groups {M}x{K}")


@pytest.mark.parametrize("N,K", [(128, 128), (300, 256), (1000, 384), (64, 512)])
def test_blocks_bit_exact(N, K):
    w = synth.make_w(N, K, seed=N + K)
    q, s = fq.fp8_quant_weight(w.to(DEV), fq.BLOCK128)
    rq, rs = oracle.quant_blocks128(w)
    assert tuple(s.shape) == ((N + 127) // 128, K // 128)
    P.assert_codes_equal(q, rq, f"blocks {N}x{K}")
    P.assert_scales_equal(s, rs, f"blocks {N}x{K}")


def test_channel_weight_is_per_row():
    w = synth.make_w(777, 512, seed=3)
    q, s = fq.fp8_quant_weight(w.to(DEV), fq.CHANNEL_TOKEN)
    rq, rs = oracle.quant_rows(w)
    P.assert_codes_equal(q, rq, "channel weight")
    P.assert_scales_equal(s, rs, "channel weight")


def test_special_values():
    K = 256
    x = torch.zeros(8, K, dtype=torch.bfloat16)
    x[1, 3] = -0.0                        # only a negative zero
    x[2, :] = 1e-30                       # everything tiny (scale ~2e-33)
    x[3, 0] = 3.0e38                      # huge amax, the rest flushed to +-0
    x[3, 1:] = -1.0
    x[4, :] = torch.linspace(-448, 448, K)
    x[5, ::2] = 1.0
    x[5, 1::2] = -1.0
    x[6, 7] = 2.0 ** -133                 # smallest bf16 subnormal as the amax
    x[7] = synth.make_x(1, K, seed=9)[0]
    x[7, 5] = -x[7].abs().max()           # negative amax
    for mode in (fq.CHANNEL_TOKEN, fq.BLOCK128):
        q, s = fq.fp8_quant_act(x.to(DEV), mode)
        rq, rs = oracle.quant_act(x, mode)
        P.assert_codes_equal(q, rq, f"special mode {mode}")
        P.assert_scales_equal(s, rs, f"special mode {mode}")


def test_strided_input_and_output():
    M, K = 37, 384
    big = synth.make_x(M, 1024, seed=5).to(DEV)
    x = big[:, 128:128 + K]               # row stride 1024 elements
    qbuf = torch.full((M, 512), 0xAB, dtype=torch.uint8, device=DEV)
    q = qbuf[:, :K]
    s = torch.empty(M, dtype=torch.float32, device=DEV)
    fq.fp8_quant_act(x, fq.CHANNEL_TOKEN, out=(q, s))
    rq, rs = oracle.quant_rows(x.cpu().contiguous())
    P.assert_codes_equal(q, rq, "strided")
    P.assert_scales_equal(s, rs, "strided")
    assert torch.all(qbuf[:, K:] == 0xAB)     # nothing written past K


def test_empty_rows():
    x = torch.empty(0, 256, dtype=torch.bfloat16, device=DEV)
    q, s = fq.fp8_quant_act(x)
    assert q.shape == (0, 256) and s.shape == (0,)


def test_every_bf16_pair_matches_ieee_division():
    """The quantizer's division (reciprocal + correction step) against torch's
    IEEE fp32 division and fp8 cast, for every positive finite bf16 amax and
    every bf16 x with |x| <= amax (both signs, zeros and subnormals included).
    Row r holds amax_r first, then all 65536 bf16 patterns with those above
    amax_r replaced by 0."""
    allv = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).to(DEV)
    finite = torch.isfinite(allv.float())
    allv = torch.where(finite, allv, torch.zeros_like(allv))
    amax_bits = torch.arange(1, 0x7F80, dtype=torch.int32, device=DEV)   # +subnormals .. max finite
    K = 65536 + 16
    chunk = 1024
    for lo in range(0, amax_bits.numel(), chunk):
        a = amax_bits[lo:lo + chunk].to(torch.int16).view(torch.bfloat16)
        R = a.numel()
        x = torch.zeros((R, K), dtype=torch.bfloat16, device=DEV)
        x[:, 0] = a
        keep = allv.float().abs()[None, :] <= a.float()[:, None]
        x[:, 16:] = torch.where(keep, allv[None, :], torch.zeros((), dtype=torch.bfloat16, device=DEV))
        q, s = fq.fp8_quant_act(x, fq.CHANNEL_TOKEN)
        # tensor / tensor: an elementwise IEEE division (dividing by a CPU scalar
        # would become a multiplication by its reciprocal)
        s_ref = a.float() / torch.full((R,), 448.0, device=DEV)
        q_ref = (x.float() / s_ref[:, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        assert torch.equal(s.view(torch.int32), s_ref.view(torch.int32)), f"scales differ in rows {lo}.."
        bad = (q != q_ref)
        if bad.any():
            r, c = bad.nonzero()[0].tolist()
            raise AssertionError(f"amax {float(a[r])}: x {float(x[r, c])} gives {int(q[r, c]):#04x}, "
                                 f"IEEE division {int(q_ref[r, c]):#04x} ({int(bad.sum())} differ in this chunk)")


def test_groups_every_bf16_pair_matches_ieee_division():
    """The per-128-group quantizer (scale and reciprocal from tables of the
    amax's mantissa for amax >= 2^-117, by division below) against torch's IEEE
    fp32 division and fp8 cast: for every positive finite bf16 amax, groups
    holding amax first and then every bf16 x with |x| <= amax (127 per group,
    both signs, zeros and subnormals included)."""
    allv = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).to(DEV)
    allv = torch.where(torch.isfinite(allv.float()), allv, torch.zeros_like(allv))
    amax_bits = torch.arange(1, 0x7F80, dtype=torch.int32, device=DEV)   # +subnormals .. max finite
    G = -(-65536 // 127)                                                  # groups per amax
    pad = G * 127 - 65536
    chunk = 512
    for lo in range(0, amax_bits.numel(), chunk):
        a = amax_bits[lo:lo + chunk].to(torch.int16).view(torch.bfloat16)
        R = a.numel()
        keep = allv.float().abs()[None, :] <= a.float()[:, None]
        vals = torch.where(keep, allv[None, :], torch.zeros((), dtype=torch.bfloat16, device=DEV))
        vals = torch.cat([vals, torch.zeros((R, pad), dtype=torch.bfloat16, device=DEV)], dim=1).view(R, G, 127)
        x = torch.cat([a.view(R, 1, 1).expand(R, G, 1), vals], dim=2).reshape(R, G * 128)
        q, s = fq.fp8_quant_act(x, fq.BLOCK128)
        s_ref = (a.float() / torch.full((R,), 448.0, device=DEV))[:, None].expand(R, G)
        assert torch.equal(s.view(torch.int32), s_ref.contiguous().view(torch.int32)), f"scales differ in rows {lo}.."
        q_ref = (x.float().view(R, G, 128) / s_ref[:, :, None]).to(torch.float8_e4m3fn).view(torch.uint8).view(R, -1)
        bad = q != q_ref
        if bad.any():
            r, c = bad.nonzero()[0].tolist()
            raise AssertionError(f"amax {float(a[r])}: x {float(x[r, c])} gives {int(q[r, c]):#04x}, "
                                 f"IEEE division {int(q_ref[r, c]):#04x} ({int(bad.sum())} differ in this chunk)")


@pytest.mark.parametrize("T,H", [(1, 8), (37, 8), (8192, 8), (513, 2)])
def test_kv_cache_per_token_per_head(T, H):
    # one scale per (token, head) of a [T, H, 128] K or V tensor: each head is a
    # 128-group of the [T, H*128] rows
    kv = synth.make_x(T, H * 128, seed=T + H)
    q, s = fq.fp8_quant_kv(kv.view(T, H, 128).to(DEV))
    rq, rs = oracle.quant_groups128(kv)
    assert tuple(q.shape) == (T, H, 128) and tuple(s.shape) == (T, H)
    P.assert_codes_equal(q.view(T, H * 128), rq, f"kv {T}x{H}")
    P.assert_scales_equal(s, rs, f"kv {T}x{H}")


@pytest.mark.parametrize("mode", [fq.CHANNEL_TOKEN, fq.BLOCK128])
def test_bf16_scale_option_bit_exact(mode):
    # scales rounded to bf16 before the codes (the checkpoints' scale dtype)
    x = synth.make_x(300, 1024, seed=31)
    w = synth.make_w(528, 1024, seed=31)     # N % 128 = 16: a partial last weight block
    q, s = fq.fp8_quant_act(x.to(DEV), mode | fq.SCALE_BF16)
    rq, rs = oracle.quant_act(x, mode, scale_bf16=True)
    P.assert_codes_equal(q, rq, f"act bf16 scales mode {mode}")
    P.assert_scales_equal(s, rs, f"act bf16 scales mode {mode}")
    qw, sw = fq.fp8_quant_weight(w.to(DEV), mode | fq.SCALE_BF16)
    rqw, rsw = oracle.quant_weight(w, mode, scale_bf16=True)
    P.assert_codes_equal(qw, rqw, f"weight bf16 scales mode {mode}")
    P.assert_scales_equal(sw, rsw, f"weight bf16 scales mode {mode}")
    # the linear accepts the option and ignores it
    y1 = fq.fp8_linear(q, s, qw, sw, mode | fq.SCALE_BF16)
    y0 = fq.fp8_linear(q, s, qw, sw, mode)
    assert torch.equal(y0, y1)
    P.assert_y_close(y1.float().cpu().numpy(), oracle.linear(rq, rs, rqw, rsw, mode), what="linear, bf16 scales")


def test_bf16_scale_option_special_values():
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    x[1, 0] = 1632.0                             # scale rounds down: the max element saturates
    x[1, 5] = -1632.0
    x[2, 3] = 2.0 ** -133                        # scale rounds to zero: becomes 1
    x[3] = synth.make_x(1, 256, seed=4)[0]
    for mode in (fq.CHANNEL_TOKEN, fq.BLOCK128):
        q, s = fq.fp8_quant_act(x.to(DEV), mode | fq.SCALE_BF16)
        rq, rs = oracle.quant_act(x, mode, scale_bf16=True)
        P.assert_codes_equal(q, rq, f"special bf16 scales mode {mode}")
        P.assert_scales_equal(s, rs, f"special bf16 scales mode {mode}")


@pytest.mark.parametrize("M,K", [(1, 16), (37, 4096), (2048, 3072), (300, 1040)])
def test_static_scale_bit_exact(M, K):
    x = synth.make_x(M, K, seed=M * 3 + K)
    scale = oracle.percentile_scale(x)
    xd = x.to(DEV)
    assert fq.calibrate_static_scale(xd) == scale
    q, s = fq.fp8_quant_act_static(xd, scale)
    P.assert_codes_equal(q, oracle.quant_static(x, scale), f"static {M}x{K}")
    assert torch.all(s == scale)
    # the codes and the filled per-token scales go straight into the linear
    w = synth.make_w(256, K, seed=K)
    wq, ws = fq.fp8_quant_weight(w.to(DEV))
    y = fq.fp8_linear(q, s, wq, ws).float().cpu().numpy()
    rwq, rws = oracle.quant_rows(w)
    rq = oracle.quant_static(x, scale)
    P.assert_y_close(y, oracle.linear(rq, np.full(M, scale, np.float32), rwq, rws, 0), what=f"static linear {M}x{K}")


def _calib_cases():
    g = torch.Generator().manual_seed(21)
    out = {"llama 8b attn_in 8192x4096": synth.make_x(8192, 4096, seed=1),
           "mostly negative": (-synth.make_x(64, 512, seed=2).float().abs() + 0.01).to(torch.bfloat16),
           "constant": torch.full((3, 64), -2.5, dtype=torch.bfloat16),
           "zeros": torch.zeros(4, 16, dtype=torch.bfloat16),
           "one row of 8": synth.make_x(1, 8, seed=3),
           "heavy tails": (torch.randn(257, 96, generator=g) ** 3 * 1e3).to(torch.bfloat16)}
    sub = torch.zeros(8, 64, dtype=torch.bfloat16)
    sub[:, ::3] = 2.0 ** -130                    # bf16 subnormals
    sub[0, 1] = -(2.0 ** -133)
    out["subnormals"] = sub
    return out


@pytest.mark.parametrize("name", list(_calib_cases()))
@pytest.mark.parametrize("lo,hi", [(0.001, 0.999), (0.0, 1.0), (0.25, 0.5), (0.1, 0.9)])
def test_calibration_kernel_equals_the_oracle(name, lo, hi):
    # order statistics from the bit-pattern histogram, interpolated in double:
    # the same fp32 scale as the oracle's sort, bit for bit; the workspace is
    # left zero for the next call
    x = _calib_cases()[name]
    hist = torch.zeros(fq.CALIB_HIST_BINS, dtype=torch.int32, device=DEV)
    got = fq.calibrate_static_scale(x.to(DEV), lo, hi, hist=hist)
    want = oracle.percentile_scale(x, lo, hi)
    assert np.float32(got) == np.float32(want), f"{name}: {got!r} vs {want!r}"
    assert int(hist.abs().sum().item()) == 0


def test_calibration_of_a_strided_view():
    big = synth.make_x(300, 1024 + 64, seed=9)
    xd = big.to(DEV)[:, 32:32 + 1024]
    assert fq.calibrate_static_scale(xd) == oracle.percentile_scale(big[:, 32:32 + 1024].contiguous())


def test_static_scale_saturates_outliers():
    x = synth.make_x(64, 512, seed=5)            # outlier columns far above the P99.9 range
    scale = oracle.percentile_scale(x)
    q, _ = fq.fp8_quant_act_static(x.to(DEV), scale)
    ref = oracle.quant_static(x, scale)
    P.assert_codes_equal(q, ref, "static outliers")
    assert ((ref & 0x7F) == 0x7E).sum() > 0       # some elements saturate
