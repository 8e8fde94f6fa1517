"""GPU FP8 linear (tcgen05 prefill, swap-AB stream-K decode) vs the exact oracle.

Both sides start from the same bf16 inputs; each quantizes with its own code
(the codes were shown bit-exact separately), and the outputs must agree
within 4e-3 * max|y_ref| + 1 bf16 ulp elementwise.
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


def run_gpu(x, w, mode, ldy_pad=0):
    xd, wd = x.to(DEV), w.to(DEV)
    wq, ws = fq.fp8_quant_weight(wd, mode)
    xq, xs = fq.fp8_quant_act(xd, mode)
    M, N = x.shape[0], w.shape[0]
    out = None
    if ldy_pad:
        full = torch.full((M, N + ldy_pad), 7.0, dtype=torch.bfloat16, device=DEV)
        out = full[:, :N]
    y = fq.fp8_linear(xq, xs, wq, ws, mode, out=out)
    torch.cuda.synchronize()
    if ldy_pad:
        assert torch.all(full[:, N:] == 7.0), "columns past N were written"
    return y, (xq, xs, wq, ws)


def check_full(M, N, K, mode, seed=0, ldy_pad=0):
    x = synth.make_x(M, K, seed=seed)
    w = synth.make_w(N, K, seed=seed)
    y, (xq, xs, wq, ws) = run_gpu(x, w, mode, ldy_pad)
    rxq, rxs = oracle.quant_act(x, mode)
    rwq, rws = oracle.quant_weight(w, mode)
    P.assert_codes_equal(xq, rxq, "xq")
    P.assert_codes_equal(wq, rwq, "wq")
    yref = oracle.linear(rxq, rxs, rwq, rws, mode)
    P.assert_y_close(y.float().cpu().numpy(), yref, what=f"Y {M}x{N}x{K} mode {mode}")
    return y


# ----------------------------------------------------------- prefill path ---

@pytest.mark.parametrize("M,N,K", [
    (65, 16, 16),          # smallest prefill problem: one partial tile everywhere
    (200, 320, 272),       # ragged M, N (BN=256) and K (128-byte blocks)
    (129, 512, 256),
    (384, 768, 1024),      # CTA-pair kernel (M >= 256), several tiles, 8 K blocks
    (300, 320, 272),       # pair kernel with a second 256-row tile mostly past M
    (1000, 1040, 400),     # pair kernel, ragged in M, N and K
    (2048, 2560, 256),     # more tiles than pairs: persistent loop, tail split in N halves
])
def test_prefill_channel(M, N, K):
    check_full(M, N, K, fq.CHANNEL_TOKEN, seed=M)


@pytest.mark.parametrize("kernel,M,N,K,mode", [("single", 2048, 2560, 256, 0), ("single", 1024, 4096, 512, 0),
                                               ("pair", 200, 320, 272, 0), ("pair", 65, 512, 128, 0),
                                               ("single", 1024, 3072, 512, 1), ("pair", 200, 384, 384, 1),
                                               ("pair", 65, 272, 128, 1)])
def test_prefill_kernel_forced(kernel, M, N, K, mode):
    # each prefill kernel on shapes the default dispatch would give the other one
    import os
    import subprocess
    import sys
    env = dict(os.environ, FP8Q_PREFILL_KERNEL=kernel)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-m", "tests._forced_kernel", str(M), str(N), str(K), str(mode)],
                       cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr


@pytest.mark.parametrize("M,N,K", [
    (512, 10240, 1024),    # 80 tiles on the pairs: the default schedule is stream-K
    (8192, 1024, 512),     # 128 tiles (the Llama-3.1-8B k/v_proj shape, shorter K)
    (300, 2560, 640),      # tiles cut at K blocks that are not tile boundaries, a ragged second row-tile
    (1000, 1040, 400),     # ragged M, N and K
])
def test_prefill_streamk(M, N, K):
    # the stream-K pair schedule (parts of tiles summed by the last pair to
    # finish), forced on, against the oracle; repeated with the same workspace:
    # its counters are left zero
    import os
    import subprocess
    import sys
    env = dict(os.environ, FP8Q_PREFILL_STREAMK="1", FP8Q_PREFILL_KERNEL="pair")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-m", "tests._forced_kernel", "streamk", str(M), str(N), str(K)],
                       cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr


def test_prefill_needs_no_workspace_by_default():
    # stream-K is opt-in (FP8Q_PREFILL_STREAMK=1): by default no prefill shape asks for scratch
    for M, N, K in ((512, 10240, 8192), (8192, 1024, 4096), (8192, 4096, 4096)):
        assert fq.fp8_linear_workspace_size(M, N, K, fq.CHANNEL_TOKEN) == 0
        assert fq.fp8_linear_workspace_size(M, N, K, fq.BLOCK128) == 0


def test_streamk_falls_back_without_a_workspace():
    # forced on, but no workspace (or a short one): the data-parallel schedule runs
    import os
    import subprocess
    import sys
    env = dict(os.environ, FP8Q_PREFILL_STREAMK="1")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-m", "tests._forced_kernel", "streamk_fallback"],
                       cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr


@pytest.mark.parametrize("M,N,K", [
    (200, 384, 384),
    (130, 144, 256),       # a partial 128-row weight block
    (256, 256, 128),       # CTA-pair kernel (M >= 256): one tile, one K block
    (300, 384, 384),       # pair kernel: second tile half past N (its second weight block absent)
    (1000, 1040, 512),     # pair kernel, ragged M and a 16-row last weight block
    (1024, 3072, 512),     # pair kernel, 48 tiles
    (2048, 2560, 256),     # more tiles than pairs: persistent loop, tail split into 128-column halves
    (4096, 1024, 1152),    # 9 K blocks: slots wrap over an odd number of K blocks per tile
])
def test_prefill_block(M, N, K):
    check_full(M, N, K, fq.BLOCK128, seed=N)




@pytest.mark.parametrize("mode", [0, 1])
def test_prefill_output_stride(mode):
    check_full(150, 256, 256, mode, ldy_pad=64)
    check_full(300, 272, 384, mode, ldy_pad=40)


# ------------------------------------------------------------ decode path ---

@pytest.mark.parametrize("M", [1, 2, 8, 16, 17, 31, 32, 33, 64])
def test_decode_channel_stream_k(M):
    # 8 weight tiles x 32 K blocks = 256 steps over at most 148 CTAs: segments
    # cross tile boundaries
    check_full(M, 1024, 4096, fq.CHANNEL_TOKEN, seed=M)


@pytest.mark.parametrize("M,N,K", [(1, 400, 1040), (5, 16, 16), (64, 4096, 128)])
def test_decode_channel_ragged(M, N, K):
    check_full(M, N, K, fq.CHANNEL_TOKEN, seed=N)


@pytest.mark.parametrize("M,N,K,mode", [
    (1, 10240, 1024, fq.CHANNEL_TOKEN),    # 80 tiles, 8 K blocks: 160 CTAs of half a tile each
    (16, 11776, 512, fq.CHANNEL_TOKEN),    # 92 tiles: 184 CTAs of half a tile
    (8, 8192, 1536, fq.CHANNEL_TOKEN),     # 64 tiles, 12 K blocks: 192 CTAs of a third of a tile
    (1, 8192, 512, fq.CHANNEL_TOKEN),      # 64 tiles, 4 K blocks (3 does not divide): 256 CTAs of one K block
    (8, 10240, 1152, fq.CHANNEL_TOKEN),    # 80 tiles, 9 K blocks (odd): 240 CTAs of a third of a tile
    (8, 10240, 896, fq.CHANNEL_TOKEN),     # 7 K blocks: no c divides them at two CTAs per SM, one CTA per SM
    (1, 10240, 1024, fq.BLOCK128),         # block scales on 160 CTAs, summed by the reduction kernel
])
def test_decode_tile_aligned_grid(M, N, K, mode):
    # two CTAs per SM for 16-token tiles: where c CTAs per weight tile (c
    # dividing the K blocks) fill the SMs at no more than two per SM, every
    # CTA streams exactly 1/c of one tile
    check_full(M, N, K, mode, seed=N + K)


@pytest.mark.parametrize("M,N,K", [(1, 272, 384), (16, 1024, 2048), (40, 512, 1024), (64, 256, 128)])
def test_decode_block(M, N, K):
    check_full(M, N, K, fq.BLOCK128, seed=K)


def test_decode_output_stride():
    check_full(3, 512, 512, fq.CHANNEL_TOKEN, ldy_pad=32)


@pytest.mark.parametrize("M,N,K,mode", [
    (1, 128, 65536, fq.CHANNEL_TOKEN),   # one weight tile, 512 K blocks over every SM: ~148 segments to add
    (3, 256, 8192, fq.CHANNEL_TOKEN),    # 128 steps < SMs: one step per CTA, 64 segments per tile
    (2, 128, 32768, fq.BLOCK128),        # block mode, one tile split over every SM
])
def test_decode_many_segments_per_tile(M, N, K, mode):
    check_full(M, N, K, mode, seed=K)


@pytest.mark.parametrize("sums,M,N,K,mode", [
    ("cluster", 1, 272, 384, fq.BLOCK128),        # 3 weight tiles of 3 K blocks: clusters of 3, one K block a CTA
    ("cluster", 16, 1024, 2048, fq.BLOCK128),     # 8 tiles of 16 K blocks: clusters of 8
    ("cluster", 3, 8192, 3072, fq.BLOCK128),      # the Llama-3.2-3B gate/up_proj shape (the default picks clusters)
    ("cluster", 33, 3072, 8192, fq.BLOCK128),     # down_proj: 24 tiles, 64 K blocks, 64-token tile
    ("cluster", 40, 528, 1040, fq.CHANNEL_TOKEN),  # channel scales, ragged N and K
    ("cluster", 5, 304, 1024, fq.CHANNEL_TOKEN),   # a partial last weight tile
    ("cluster", 64, 256, 128, fq.BLOCK128),       # one K block: no cluster fits, the default path runs
    ("kernel", 16, 1024, 2048, fq.BLOCK128),      # block scales, summed by the last CTA to finish
    ("separate", 8, 1024, 4096, fq.CHANNEL_TOKEN),  # channel scales, summed by the reduction kernel
    ("separate", 16, 8192, 3072, fq.BLOCK128),
])
def test_decode_sums_forced(sums, M, N, K, mode):
    # each place the split weight tiles can be summed, forced on shapes the
    # default dispatch may give another; three calls on one workspace
    import os
    import subprocess
    import sys
    env = dict(os.environ, FP8Q_DECODE_SUMS=sums)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-m", "tests._forced_kernel", "decode", str(M), str(N), str(K), str(mode)],
                       cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr


@pytest.mark.parametrize("env,M,N,K,mode", [
    ({"FP8Q_DECODE_STAGES": "full"}, 8, 4096, 4096, fq.CHANNEL_TOKEN),   # 16-token tiles, one CTA per SM
    ({"FP8Q_DECODE_STAGES": "full"}, 16, 8192, 3072, fq.BLOCK128),       # ... on the cluster path
    ({"FP8Q_DECODE_STAGES": "half"}, 32, 2048, 4096, fq.CHANNEL_TOKEN),  # 32-token tiles, two CTAs per SM
    ({"FP8Q_DECODE_STAGES": "half"}, 64, 1024, 8192, fq.CHANNEL_TOKEN),  # 64-token tiles, two CTAs per SM
    ({"FP8Q_DECODE_EARLY": "1"}, 1, 10240, 8192, fq.CHANNEL_TOKEN),      # early loads where ranges are shorter than a tile
    ({"FP8Q_DECODE_EARLY": "0"}, 8, 20480, 1024, fq.CHANNEL_TOKEN),      # none where they are longer
    ({"FP8Q_DECODE_EARLY": "1", "FP8Q_DECODE_STAGES": "full"}, 4, 10240, 8192, fq.CHANNEL_TOKEN),
])
def test_decode_builds_forced(env, M, N, K, mode):
    # the decode kernel's other builds (one or two CTAs per SM, early loads of
    # a known last contributor on or off), forced on shapes the default
    # dispatch gives another; three calls on one workspace
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-m", "tests._forced_kernel", "decode", str(M), str(N), str(K), str(mode)],
                       cwd=root, env=dict(os.environ, **env), capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr


def test_decode_workspace_left_reusable():
    # The workspace is all zero again after every call, so one zero-filled
    # buffer serves calls of different shapes and modes in a row (a later call
    # may put its arrival counters where an earlier one kept partial sums).
    size = max(fq.fp8_linear_workspace_size(M, N, K, mode)
               for M, N, K, mode in [(1, 4096, 4096, 0), (16, 1024, 2048, 1), (64, 512, 8192, 0)])
    wsp = torch.zeros(size, dtype=torch.uint8, device=DEV)
    for M, N, K, mode in [(1, 4096, 4096, 0), (16, 1024, 2048, 1), (64, 512, 8192, 0), (1, 4096, 4096, 0)]:
        x = synth.make_x(M, K, seed=N)
        w = synth.make_w(N, K, seed=N)
        wq, ws = fq.fp8_quant_weight(w.to(DEV), mode)
        xq, xs = fq.fp8_quant_act(x.to(DEV), mode)
        y = fq.fp8_linear(xq, xs, wq, ws, mode, workspace=wsp).float().cpu().numpy()
        rxq, rxs = oracle.quant_act(x, mode)
        rwq, rws = oracle.quant_weight(w, mode)
        P.assert_y_close(y, oracle.linear(rxq, rxs, rwq, rws, mode), what=f"reused workspace {M}x{N}x{K} m{mode}")
        assert torch.count_nonzero(wsp).item() == 0, "workspace not left zero"


def test_zero_activations_give_zero():
    x = torch.zeros(70, 256, dtype=torch.bfloat16)
    w = synth.make_w(128, 256)
    for M in (70, 4):
        y, _ = run_gpu(x[:M], w, fq.CHANNEL_TOKEN)
        assert torch.all(y == 0)


def test_empty_m():
    xq = torch.empty(0, 256, dtype=torch.uint8, device=DEV)
    xs = torch.empty(0, dtype=torch.float32, device=DEV)
    wq = torch.zeros(64, 256, dtype=torch.uint8, device=DEV)
    ws = torch.ones(64, dtype=torch.float32, device=DEV)
    assert fq.fp8_linear(xq, xs, wq, ws).shape == (0, 64)


def test_workspace_too_small_is_rejected():
    xq = torch.zeros(4, 256, dtype=torch.uint8, device=DEV)
    xs = torch.ones(4, dtype=torch.float32, device=DEV)
    wq = torch.zeros(256, 256, dtype=torch.uint8, device=DEV)
    ws = torch.ones(256, dtype=torch.float32, device=DEV)
    small = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(fq.FP8QError) as e:
        fq.fp8_linear(xq, xs, wq, ws, workspace=small)
    assert e.value.status == fq.ERR_INVALID_ARG


def test_repeat_calls_are_deterministic():
    x = synth.make_x(8, 2048, seed=3).to(DEV)
    w = synth.make_w(2048, 2048, seed=3).to(DEV)
    wq, ws = fq.fp8_quant_weight(w)
    xq, xs = fq.fp8_quant_act(x)
    y0 = fq.fp8_linear(xq, xs, wq, ws)
    for _ in range(3):
        assert torch.equal(fq.fp8_linear(xq, xs, wq, ws), y0)


# Every workload at full size (every code and scale, outputs on sampled rows
# and weight blocks) is in test_gpu_full_size.py.

ALL = synth.workloads()


def test_tiny_workload_in_full():
    g = ALL["tiny_16x256x512"].gemms[0]
    x = synth.make_x(g.M, g.K, seed=0, n_out=2)
    w = synth.make_w(g.N, g.K, seed=0)
    y, (xq, xs, wq, ws) = run_gpu(x, w, fq.CHANNEL_TOKEN)
    rxq, rxs = oracle.quant_rows(x)
    rwq, rws = oracle.quant_rows(w)
    P.assert_codes_equal(xq, rxq, "tiny xq")
    P.assert_scales_equal(xs, rxs, "tiny xs")
    P.assert_codes_equal(wq, rwq, "tiny wq")
    P.assert_scales_equal(ws, rws, "tiny ws")
    P.assert_y_close(y.float().cpu().numpy(), oracle.linear(rxq, rxs, rwq, rws, 0), what="tiny")


@pytest.mark.parametrize("M,mode", [(4, fq.CHANNEL_TOKEN), (300, fq.CHANNEL_TOKEN), (16, fq.BLOCK128),
                                    (256, fq.BLOCK128)])
def test_cuda_graph_replay_matches_eager(M, mode):
    N, K = 1024, 1024
    x = synth.make_x(M, K, seed=M).to(DEV)
    w = synth.make_w(N, K, seed=M).to(DEV)
    wq, ws = fq.fp8_quant_weight(w, mode)
    xq, xs = fq.fp8_quant_act(x, mode)
    y_eager = fq.fp8_linear(xq, xs, wq, ws, mode)
    xq2, xs2 = torch.empty_like(xq), torch.empty_like(xs)
    y2 = torch.empty_like(y_eager)
    wsp = torch.zeros(max(1, fq.fp8_linear_workspace_size(M, N, K, mode)), dtype=torch.uint8, device=DEV)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            fq.fp8_quant_act(x, mode, out=(xq2, xs2))
            fq.fp8_linear(xq2, xs2, wq, ws, mode, out=y2, workspace=wsp)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(3):
        y2.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(xq2, xq) and torch.equal(xs2, xs)
        assert torch.equal(y2, y_eager)
