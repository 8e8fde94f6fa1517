"""Run one FP8 linear with the prefill kernel forced by FP8Q_PREFILL_KERNEL
(set by the caller) and check it against the oracle.  Exit status 0 = pass.

    python -m tests._forced_kernel M N K mode

or one weight-only linear with the kernel forced by FP8Q_W8A16_KERNEL:

    python -m tests._forced_kernel w8a16 M N K

or three calls of the stream-K prefill schedule (FP8Q_PREFILL_STREAMK=1) on one
workspace, each checked against the oracle and the counters checked zero:

    python -m tests._forced_kernel streamk M N K

or three decode calls (M <= 64) with the split-tile sums forced by
FP8Q_DECODE_SUMS (separate, kernel or cluster) on one workspace, each checked
against the oracle, bit-equal to each other, the workspace left zero:

    python -m tests._forced_kernel decode M N K mode
"""
import sys

import synth
import oracle
import fp8_w8a8_quantized_amax_b200 as fq
from tests import _parity as P


def w8a16():
    M, N, K = (int(a) for a in sys.argv[2:5])
    x = synth.make_x(M, K, seed=M + N)
    w = synth.make_w(N, K, seed=M + N)
    wq, ws = oracle.quant_rows(w)
    import torch
    y = fq.fp8_linear_w8a16(x.to("cuda"), torch.from_numpy(wq).to("cuda"), torch.from_numpy(ws).to("cuda"))
    P.assert_y_close(y.float().cpu().numpy(), oracle.linear_w8a16(x, wq, ws), what=f"forced W8A16 {M}x{N}x{K}")
    assert fq.device_error(clear=True) == 0
    print("ok")


def streamk():
    import torch
    M, N, K = (int(a) for a in sys.argv[2:5])
    x = synth.make_x(M, K, seed=M + N)
    w = synth.make_w(N, K, seed=M + N)
    wq, ws = fq.fp8_quant_weight(w.to("cuda"))
    xq, xs = fq.fp8_quant_act(x.to("cuda"))
    need = fq.fp8_linear_workspace_size(M, N, K, fq.CHANNEL_TOKEN)
    assert need > 0, "stream-K was not selected"
    wk = torch.zeros(need, dtype=torch.uint8, device="cuda")
    rxq, rxs = oracle.quant_act(x, fq.CHANNEL_TOKEN)
    rwq, rws = oracle.quant_weight(w, fq.CHANNEL_TOKEN)
    yref = oracle.linear(rxq, rxs, rwq, rws, fq.CHANNEL_TOKEN)
    n_tiles = -(-M // 256) * -(-N // 256)
    ys = []
    for _ in range(3):
        y = fq.fp8_linear(xq, xs, wq, ws, workspace=wk)
        torch.cuda.synchronize()
        P.assert_y_close(y.float().cpu().numpy(), yref, what=f"stream-K {M}x{N}x{K}")
        assert int(wk[: n_tiles * 64].abs().sum().item()) == 0, "arrival counters not left zero"
        ys.append(y)
    assert all(torch.equal(ys[0], y) for y in ys[1:]), "stream-K sums are not deterministic"
    assert fq.device_error(clear=True) == 0
    print("ok")


def streamk_fallback():
    # FP8Q_PREFILL_STREAMK=1 but no workspace: the data-parallel schedule runs,
    # the same sums in another order as with the workspace
    import torch
    M, N, K = 512, 10240, 512
    x = synth.make_x(M, K, seed=1).to("cuda")
    w = synth.make_w(N, K, seed=1).to("cuda")
    wq, ws = fq.fp8_quant_weight(w)
    xq, xs = fq.fp8_quant_act(x)
    assert fq.fp8_linear_workspace_size(M, N, K, fq.CHANNEL_TOKEN) > 0
    y_sk = fq.fp8_linear(xq, xs, wq, ws)
    y_dp = torch.empty_like(y_sk)
    st = fq.lib().fp8_linear(xq.data_ptr(), xs.data_ptr(), wq.data_ptr(), ws.data_ptr(), M, N, K, 0,
                             y_dp.data_ptr(), N, None, 0, torch.cuda.current_stream().cuda_stream)
    assert st == fq.OK
    torch.cuda.synchronize()
    rxq, rxs = oracle.quant_act(x.cpu(), fq.CHANNEL_TOKEN)
    rwq, rws = oracle.quant_weight(w.cpu(), fq.CHANNEL_TOKEN)
    yref = oracle.linear(rxq, rxs, rwq, rws, fq.CHANNEL_TOKEN)
    P.assert_y_close(y_dp.float().cpu().numpy(), yref, what="data-parallel fallback")
    P.assert_y_close(y_sk.float().cpu().numpy(), yref, what="stream-K")
    assert fq.device_error(clear=True) == 0
    print("ok")


def decode():
    import torch
    M, N, K, mode = (int(a) for a in sys.argv[2:6])
    x = synth.make_x(M, K, seed=M + N)
    w = synth.make_w(N, K, seed=M + N)
    wq, ws = fq.fp8_quant_weight(w.to("cuda"), mode)
    xq, xs = fq.fp8_quant_act(x.to("cuda"), mode)
    wk = torch.zeros(fq.fp8_linear_workspace_size(M, N, K, mode), dtype=torch.uint8, device="cuda")
    rxq, rxs = oracle.quant_act(x, mode)
    rwq, rws = oracle.quant_weight(w, mode)
    yref = oracle.linear(rxq, rxs, rwq, rws, mode)
    ys = []
    for _ in range(3):
        y = fq.fp8_linear(xq, xs, wq, ws, mode, workspace=wk)
        torch.cuda.synchronize()
        P.assert_y_close(y.float().cpu().numpy(), yref, what=f"decode {M}x{N}x{K} mode {mode}")
        assert torch.count_nonzero(wk).item() == 0, "workspace not left zero"
        ys.append(y)
    assert all(torch.equal(ys[0], y) for y in ys[1:]), "decode sums are not deterministic"
    assert fq.device_error(clear=True) == 0
    print("ok")


def main():
    if sys.argv[1] == "decode":
        return decode()
    if sys.argv[1] == "w8a16":
        return w8a16()
    if sys.argv[1] == "streamk":
        return streamk()
    if sys.argv[1] == "streamk_fallback":
        return streamk_fallback()
    M, N, K, mode = (int(a) for a in sys.argv[1:5])
    x = synth.make_x(M, K, seed=M + N)
    w = synth.make_w(N, K, seed=M + N)
    wq, ws = fq.fp8_quant_weight(w.to("cuda"), mode)
    xq, xs = fq.fp8_quant_act(x.to("cuda"), mode)
    y = fq.fp8_linear(xq, xs, wq, ws, mode).float().cpu().numpy()
    rxq, rxs = oracle.quant_act(x, mode)
    rwq, rws = oracle.quant_weight(w, mode)
    P.assert_y_close(y, oracle.linear(rxq, rxs, rwq, rws, mode), what=f"forced {M}x{N}x{K}")
    assert fq.device_error(clear=True) == 0
    print("ok")


if __name__ == "__main__":
    main()
