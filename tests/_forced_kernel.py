"""Run one FP8 linear with the prefill kernel forced by FP8Q_PREFILL_KERNEL
(set by the caller) and check it against the oracle.  Exit status 0 = pass.

    python -m tests._forced_kernel M N K mode

or one weight-only linear with the kernel forced by FP8Q_W8A16_KERNEL:

    python -m tests._forced_kernel w8a16 M N K
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


def main():
    if sys.argv[1] == "w8a16":
        return w8a16()
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
