"""Failure detection on the device: a wait that runs out, and recovery.

Every mbarrier wait in the kernels is bounded: when it runs out it records
its wait site in the library's device error word, raises the CTA's abort
flag so that every other role of the CTA stops too, waits (again bounded)
for the loads and MMAs the CTA still has in flight, frees its tensor memory
and returns.  The product library's limit is 4 s, which no healthy run comes
near.  These tests use the test build of the library (libfp8q_testhooks.so:
limit 2 ms, plus a switch that makes CTA 0 of the decode kernel withhold
either one tensor-memory slot release -- the MMA warp's wait for that slot
runs out -- or its first accumulator commit -- the epilogue's wait runs out,
and the CTA never delivers its share of the split tiles).  Nothing faults or
hangs: the call returns, fp8q_device_error() names the wait site, and the
next call -- switch off, fresh workspace -- gives the product library's
output bit for bit.  The same holds for fp8_linear_noalloc, whose
in-library scratch (left with stale counters and partial sums by the failed
call) fp8q_device_error(1) zeroes.
"""
import ctypes

import pytest
import torch

import synth
import fp8_w8a8_quantized_amax_b200 as fq

pytestmark = pytest.mark.gpu
DEV = "cuda"
ERR_WAIT_EMPTY = 0x102        # the producer's wait for a free stage
ERR_WAIT_TMEM_FULL = 0x103    # an epilogue warp's wait for an accumulator
ERR_WAIT_TMEM_EMPTY = 0x104   # the MMA warp's wait for a tensor-memory slot
WITHHOLD_RELEASE, WITHHOLD_COMMIT = 1, 2
# The first wait to run out names itself.  A withheld slot release stalls the
# MMA warp, and the producer's wait for the stages that MMA would have freed
# starts at about the same time, so either may be first.
RELEASE_SITES = (ERR_WAIT_EMPTY, ERR_WAIT_TMEM_EMPTY, ERR_WAIT_TMEM_FULL)


@pytest.fixture(scope="module")
def T():
    from fp8_w8a8_quantized_amax_b200 import build
    build.build()
    lib = ctypes.CDLL(build.build_test_hooks())
    P, I = ctypes.c_void_p, ctypes.c_int64
    lib.fp8_linear.argtypes = [P, P, P, P, I, I, I, ctypes.c_int, P, I, P, ctypes.c_size_t, P]
    lib.fp8_linear.restype = ctypes.c_int
    lib.fp8_linear_noalloc.argtypes = [P, P, P, P, I, I, I, ctypes.c_int, P, I, P]
    lib.fp8_linear_noalloc.restype = ctypes.c_int
    lib.fp8_linear_workspace_size.argtypes = [I, I, I, ctypes.c_int]
    lib.fp8_linear_workspace_size.restype = ctypes.c_size_t
    lib.fp8q_device_error.argtypes = [ctypes.c_int]
    lib.fp8q_device_error.restype = ctypes.c_int
    lib.fp8q_test_withhold.argtypes = [ctypes.c_int]
    lib.fp8q_test_withhold.restype = ctypes.c_int
    assert lib.fp8q_device_error(1) == 0
    yield lib
    lib.fp8q_test_withhold(0)
    assert lib.fp8q_device_error(1) == 0
    assert fq.device_error(clear=False) == 0     # the product library saw nothing


# Shapes whose CTA 0 comes back to the withheld slot (8 slots): channel mode
# with K = 128 (every step its own tile, 16 tiles per CTA on 148 SMs), and
# block mode with 16 K blocks per CTA (148 tiles of 32 K blocks: two CTAs per
# tile, 296 in all, with 16-token tiles built for two CTAs per SM).
CASES = [(4, 128 * 148 * 16, 128, fq.CHANNEL_TOKEN), (16, 128 * 148, 4096, fq.BLOCK128)]
# Two K blocks per tile, 12 or 13 steps per CTA on 148 SMs: CTA 0's first
# segment is the first half of a tile that CTA 1 finishes, and CTA 0 has 7
# segments, so its MMA warp never waits for a slot: only the epilogue's wait
# for the withheld accumulator runs out.
SPLIT = (4, 128 * 889, 256, fq.CHANNEL_TOKEN)


def _operands(M, N, K, mode, seed=0):
    x = synth.make_x(M, K, seed=M + seed).to(DEV)
    w = synth.make_w(N, K, seed=N + seed).to(DEV)
    wq, ws = fq.fp8_quant_weight(w, mode)
    xq, xs = fq.fp8_quant_act(x, mode)
    return xq, xs, wq, ws


def _call(T, ops, mode, N, workspace=None, noalloc=False):
    xq, xs, wq, ws = ops
    M, K = xq.shape
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    s = torch.cuda.current_stream().cuda_stream
    if noalloc:
        st = T.fp8_linear_noalloc(xq.data_ptr(), xs.data_ptr(), wq.data_ptr(), ws.data_ptr(), M, N, K, mode,
                                  y.data_ptr(), N, s)
    else:
        st = T.fp8_linear(xq.data_ptr(), xs.data_ptr(), wq.data_ptr(), ws.data_ptr(), M, N, K, mode,
                          y.data_ptr(), N, workspace.data_ptr(), workspace.numel(), s)
    assert st == fq.OK, fq.status_string(st)
    return y


@pytest.mark.parametrize("M,N,K,mode", CASES, ids=["channel", "block"])
def test_wait_runs_out_and_the_next_call_is_correct(T, M, N, K, mode):
    ops = _operands(M, N, K, mode)
    ref = fq.fp8_linear(*ops, mode)                          # product library
    nws = T.fp8_linear_workspace_size(M, N, K, mode)
    assert T.fp8q_test_withhold(WITHHOLD_RELEASE) == 0
    _call(T, ops, mode, N, torch.zeros(nws, dtype=torch.uint8, device=DEV))
    site = T.fp8q_device_error(0)                             # synchronizes: the call has returned
    assert site in RELEASE_SITES, hex(site)
    assert T.fp8q_test_withhold(0) == 0
    assert T.fp8q_device_error(1) == site                     # read and clear
    assert T.fp8q_device_error(0) == 0
    y = _call(T, ops, mode, N, torch.zeros(nws, dtype=torch.uint8, device=DEV))
    torch.cuda.synchronize()
    assert T.fp8q_device_error(0) == 0
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("noalloc", [False, True], ids=["workspace", "noalloc"])
def test_undelivered_split_sums_and_recovery(T, noalloc):
    # The epilogue of CTA 0 waits for an accumulator that never comes: CTA 0
    # never adds its half of its first tile, so the tile's counters and CTA
    # 1's partial sums stay in the scratch.  After fp8q_device_error(1) (which
    # zeroes fp8_linear_noalloc's array) or with a fresh workspace, calls on
    # other operands are correct again, twice in a row.
    M, N, K, mode = SPLIT
    ops = _operands(M, N, K, mode)
    nws = T.fp8_linear_workspace_size(M, N, K, mode)
    wk = None if noalloc else torch.zeros(nws, dtype=torch.uint8, device=DEV)
    assert T.fp8q_test_withhold(WITHHOLD_COMMIT) == 0
    _call(T, ops, mode, N, workspace=wk, noalloc=noalloc)
    assert T.fp8q_test_withhold(0) == 0
    assert T.fp8q_device_error(1) == ERR_WAIT_TMEM_FULL
    for seed in (1, 2):
        ops2 = _operands(M, N, K, mode, seed=seed)
        wk2 = None if noalloc else torch.zeros(nws, dtype=torch.uint8, device=DEV)
        y = _call(T, ops2, mode, N, workspace=wk2, noalloc=noalloc)
        torch.cuda.synchronize()
        assert T.fp8q_device_error(0) == 0
        assert torch.equal(y.view(torch.int16), fq.fp8_linear(*ops2, mode).view(torch.int16)), f"seed {seed}"


# Cluster split-K (the Llama-3.2-3B FP8-Block gate/up decode shape: 64 weight
# tiles, clusters of 2 CTAs, 12 K blocks each): CTA 0, rank 0 of its cluster,
# withholds its first slot release (its MMA warp comes back to slot 0 at the
# ninth K block) or its first accumulator commit.  Its partner finishes and
# waits at the cluster barrier, which CTA 0 reaches after its own bounded
# waits have run out and its loads and MMAs have drained.
CLUSTER = (16, 8192, 3072, fq.BLOCK128)


@pytest.mark.parametrize("withhold,sites", [(WITHHOLD_RELEASE, RELEASE_SITES), (WITHHOLD_COMMIT, (ERR_WAIT_TMEM_FULL,))],
                         ids=["release", "commit"])
def test_cluster_path_wait_runs_out_and_the_next_call_is_correct(T, withhold, sites):
    M, N, K, mode = CLUSTER
    ops = _operands(M, N, K, mode)
    ref = fq.fp8_linear(*ops, mode)
    nws = T.fp8_linear_workspace_size(M, N, K, mode)
    assert T.fp8q_test_withhold(withhold) == 0
    _call(T, ops, mode, N, torch.zeros(nws, dtype=torch.uint8, device=DEV))
    site = T.fp8q_device_error(0)
    assert site in sites, hex(site)
    assert T.fp8q_test_withhold(0) == 0
    assert T.fp8q_device_error(1) == site
    for seed in (0, 1):
        ops2 = ops if seed == 0 else _operands(M, N, K, mode, seed=seed)
        y = _call(T, ops2, mode, N, torch.zeros(nws, dtype=torch.uint8, device=DEV))
        torch.cuda.synchronize()
        assert T.fp8q_device_error(0) == 0
        want = ref if seed == 0 else fq.fp8_linear(*ops2, mode)
        assert torch.equal(y.view(torch.int16), want.view(torch.int16)), f"seed {seed}"
