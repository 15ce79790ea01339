"""The allocation-free forward gives the same results as the forward with a workspace.

bitlinear_forward_noalloc serves callers that cannot allocate device memory
(where cudaMalloc is off limits because it can synchronise the device, or
inside an engine that owns all device memory and offers no allocator).  It
keeps its scratch in one fixed array in device memory instead of a caller
workspace.  This test calls it through the C ABI, twice in a row on the
same inputs, and checks each call against bitlinear_forward: the int32
accumulators bit for bit, the outputs within the bars every parity test
uses (fp32 within 1e-6 relative, bf16 within one ulp).  The file is named to
run after the other tests; it also runs on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import ternary_weight_a8_b200 as tb
from parity import activations, dev, weights

pytestmark = pytest.mark.gpu


def _noalloc():
    fn = tb.lib().bitlinear_forward_noalloc
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, i32, i32, vp, i32, i32, vp, i32, vp, vp]
    fn.restype = i32
    return fn


def _close(y, y_ref):
    if y.dtype == torch.float32:
        a, b = y.cpu().numpy().astype(np.float64), y_ref.cpu().numpy().astype(np.float64)
        assert (np.abs(a - b) <= 1e-6 * np.abs(b)).all()
    else:
        a = y.view(torch.int16).cpu().numpy().astype(np.int32)
        b = y_ref.view(torch.int16).cpu().numpy().astype(np.int32)
        a = np.where(a < 0, -(a & 0x7FFF), a)
        b = np.where(b < 0, -(b & 0x7FFF), b)
        assert np.abs(a - b).max(initial=0) <= 1


CASES = [  # (M, N, K, x dtype, y dtype): decode with in-kernel quantisation, decode, prefill
    (1, 6912, 2560, "bf16", torch.bfloat16),
    (8, 3200, 8640, "bf16", torch.float32),
    (64, 640, 1024, "f32", torch.float32),
]


@pytest.mark.parametrize("M,N,K,xdt,ydt", CASES)
def test_noalloc_forward_matches_workspace_forward(M, N, K, xdt, ydt):
    fn = _noalloc()
    packed, gamma = tb.pack_weights(dev(weights(N, K, seed=M + N)))
    x, _ = activations(M, K, seed=K + M, dtype=xdt)
    y_ref, acc_ref = tb.forward(packed, gamma, x, out_dtype=ydt, acc_out=True)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):  # two calls in a row share the fixed scratch
        y = torch.full((M, N), 7.0, dtype=ydt, device="cuda")
        acc = torch.full((M, N), 12345, dtype=torch.int32, device="cuda")
        rc = fn(ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(gamma.data_ptr()), N, K,
                ctypes.c_void_p(x.data_ptr()), tb.BL_BF16 if xdt == "bf16" else tb.BL_F32, M,
                ctypes.c_void_p(y.data_ptr()), tb.BL_BF16 if ydt == torch.bfloat16 else tb.BL_F32,
                ctypes.c_void_p(acc.data_ptr()), stream)
        assert rc == tb.BL_OK, tb.last_error()
        torch.cuda.synchronize()
        assert torch.equal(acc, acc_ref)
        _close(y, y_ref)


def test_noalloc_refuses_calls_larger_than_its_scratch():
    fn = _noalloc()
    M, N, K = 2048, 256, 2560  # needs about 5 MiB of scratch
    packed, gamma = tb.pack_weights(dev(weights(N, K, seed=1)))
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    rc = fn(ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(gamma.data_ptr()), N, K,
            ctypes.c_void_p(x.data_ptr()), tb.BL_BF16, M, ctypes.c_void_p(y.data_ptr()), tb.BL_BF16, None,
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == tb.BL_ERR_WORKSPACE_TOO_SMALL
    assert "fixed scratch" in tb.last_error()
