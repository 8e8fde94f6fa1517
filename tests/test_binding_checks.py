"""The binding's checks on the tensors it hands to the library, on the CPU.

A scale vector, output or workspace on the host (or of the wrong type, size
or device) would reach a kernel as a bad pointer; the binding refuses it
with ValueError before any library call.  No GPU exists here, so the CUDA
tensors are stand-ins that carry only the metadata the binding reads, and the
library is a recorder."""
import pytest
import torch

import fp8_w8a8_quantized_amax_b200 as fq

CUDA0 = torch.device("cuda", 0)
CUDA1 = torch.device("cuda", 1)


class T:
    """Metadata-only stand-in for a torch tensor."""

    def __init__(self, shape, dtype, device=CUDA0, strides=None, contiguous=True):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = device
        self.is_cuda = device.type == "cuda"
        self._contig = contiguous
        if strides is None:
            strides, acc = [], 1
            for d in reversed(shape):
                strides.insert(0, acc)
                acc *= max(d, 1)
        self._strides = tuple(strides)

    def dim(self):
        return len(self.shape)

    def stride(self, i):
        return self._strides[i]

    def numel(self):
        n = 1
        for d in self.shape:
            n *= d
        return n

    def is_contiguous(self):
        return self._contig

    def element_size(self):
        return {torch.uint8: 1, torch.bfloat16: 2, torch.float32: 4}[self.dtype]

    def data_ptr(self):
        return 0x10000


class Lib:
    def __init__(self, ws_bytes=0):
        self.calls = []
        self.ws_bytes = ws_bytes

    def __getattr__(self, name):
        def f(*args):
            self.calls.append(name)
            return self.ws_bytes if name.endswith("workspace_size") else 0
        return f


@pytest.fixture
def lib(monkeypatch):
    L = Lib()
    monkeypatch.setattr(fq, "lib", lambda: L)
    monkeypatch.setattr(fq, "_stream", lambda t: 0)
    return L


U8, BF, F32 = torch.uint8, torch.bfloat16, torch.float32


def linear_args(M=4, N=64, K=256, mode=fq.CHANNEL_TOKEN):
    channel = (mode & ~fq.SCALE_BF16) == fq.CHANNEL_TOKEN
    xs = (M,) if channel else (M, K // 128)
    ws = (N,) if channel else ((N + 127) // 128, K // 128)
    return dict(Xq=T((M, K), U8), x_scale=T(xs, F32), Wq=T((N, K), U8), w_scale=T(ws, F32), mode=mode,
                out=T((M, N), BF))


@pytest.mark.parametrize("mode", [fq.CHANNEL_TOKEN, fq.BLOCK128, fq.CHANNEL_TOKEN | fq.SCALE_BF16])
def test_linear_valid_call_reaches_the_library(lib, mode):
    fq.fp8_linear(**linear_args(mode=mode))
    assert lib.calls[-1] == "fp8_linear"


@pytest.mark.parametrize("name,bad", [
    ("x_scale", T((4,), F32, device=torch.device("cpu"))),     # host memory
    ("x_scale", T((4,), BF)),                                  # wrong type
    ("x_scale", T((3,), F32)),                                 # too small
    ("x_scale", T((4,), F32, contiguous=False)),
    ("x_scale", T((4,), F32, device=CUDA1)),                   # another GPU
    ("w_scale", T((64,), F32, device=torch.device("cpu"))),
    ("w_scale", T((63,), F32)),
    ("out", T((4, 64), F32)),
    ("out", T((4, 65), BF)),
    ("out", T((4, 64), BF, strides=(128, 2))),
    ("out", T((4, 64), BF, device=torch.device("cpu"))),
])
def test_linear_refuses_bad_tensors(lib, name, bad):
    a = linear_args()
    a[name] = bad
    with pytest.raises(ValueError):
        fq.fp8_linear(**a)
    assert "fp8_linear" not in lib.calls


def test_linear_block_scales_must_cover_every_block(lib):
    a = linear_args(mode=fq.BLOCK128)
    a["x_scale"] = T((4,), F32)                  # per-token size given for per-group scales
    with pytest.raises(ValueError):
        fq.fp8_linear(**a)


def test_linear_workspace_device_checked_size_left_to_the_library(lib):
    a = linear_args()
    with pytest.raises(ValueError):
        fq.fp8_linear(**a, workspace=T((1 << 20,), U8, device=torch.device("cpu")))
    with pytest.raises(ValueError):
        fq.fp8_linear(**a, workspace=T((1 << 18,), F32))
    fq.fp8_linear(**a, workspace=T((16,), U8))   # too small: the library's FP8Q_ERR_INVALID_ARG
    assert lib.calls[-1] == "fp8_linear"


def test_quant_outputs_checked(lib):
    X = T((8, 256), BF)
    fq.fp8_quant_act(X, out=(T((8, 256), U8), T((8,), F32)))
    fq.fp8_quant_act(X, fq.BLOCK128, out=(T((8, 256), U8, strides=(512, 1)), T((8, 2), F32)))   # strided codes
    assert lib.calls.count("fp8_quant_act") == 2
    with pytest.raises(ValueError):                   # codes of the wrong shape
        fq.fp8_quant_act(X, fq.BLOCK128, out=(T((8, 512), U8), T((8, 2), F32)))
    for bad in [(T((8, 256), U8), T((8,), F32, device=torch.device("cpu"))),
                (T((8, 256), U8), T((7,), F32)),
                (T((8, 256), BF), T((8,), F32)),
                (T((8, 256), U8), T((8, 1), F32))]:     # group scales too few
        mode = fq.BLOCK128 if bad[1].shape == torch.Size((8, 1)) else fq.CHANNEL_TOKEN
        with pytest.raises(ValueError):
            fq.fp8_quant_act(X, mode, out=bad)
    W = T((256, 256), BF)
    fq.fp8_quant_weight(W, fq.BLOCK128, out=(T((256, 256), U8), T((2, 2), F32)))
    with pytest.raises(ValueError):
        fq.fp8_quant_weight(W, fq.BLOCK128, out=(T((256, 256), U8), T((2,), F32)))


def test_fused_and_weight_only_entry_points_checked(lib):
    M, N, K = 4, 64, 256
    xq, xs, wq, ws = T((M, K), U8), T((M,), F32), T((N, K), U8), T((N,), F32)
    fq.fp8_linear_swiglu(xq, xs, wq, ws, wq, ws, out=T((M, N), BF))
    assert lib.calls[-1] == "fp8_linear_swiglu"
    with pytest.raises(ValueError):
        fq.fp8_linear_swiglu(xq, xs, wq, ws, wq, T((N,), F32, device=torch.device("cpu")), out=T((M, N), BF))
    X = T((M, K), BF)
    fq.fp8_linear_w8a16(X, wq, ws, out=T((M, N), BF), workspace=T((1 << 16,), U8))
    assert lib.calls[-1] == "fp8_linear_w8a16"
    for kw in [dict(w_scale=T((N,), F32, device=torch.device("cpu"))), dict(w_scale=T((N - 1,), F32)),
               dict(out=T((M, N), F32)), dict(workspace=T((64,), U8, device=CUDA1))]:
        a = dict(w_scale=ws, out=T((M, N), BF), workspace=T((1 << 16,), U8))
        a.update(kw)
        with pytest.raises(ValueError):
            fq.fp8_linear_w8a16(X, wq, **a)
    g = T((K,), BF)
    fq.fp8_rmsnorm_quant_act(X, g, out=(T((M, K), U8), T((M,), F32)))
    with pytest.raises(ValueError):
        fq.fp8_rmsnorm_quant_act(X, T((K,), BF, device=CUDA1), out=(T((M, K), U8), T((M,), F32)))
    with pytest.raises(ValueError):
        fq.fp8_rmsnorm_quant_act(X, g, out=(T((M, K), U8), T((M,), BF)))
    fq.fp8_quant_act_static(X, 0.1, out=(T((M, K), U8), None))      # the scale vector is optional
    with pytest.raises(ValueError):
        fq.fp8_quant_act_static(X, 0.1, out=(T((M, K), U8), T((M,), F32, device=torch.device("cpu"))))
