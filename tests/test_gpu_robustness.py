"""Failure handling on the GPU without faulting it.

Bad arguments come back as status codes before anything is launched (host
pointers, misaligned pointers, short workspaces).  The device-side bounded
wait is exercised by a barrier that nothing completes, with a limit of a few
milliseconds: the kernel gives up, records the timeout in the workspace
status word and returns, and the context stays usable.  Canary bytes around
output buffers show that kernels write nothing outside their outputs.
"""
import ctypes

import numpy as np
import pytest
import torch

import ternary_weight_a8_b200 as tb
from parity import activations, dev, weights

pytestmark = pytest.mark.gpu


def test_host_pointer_is_rejected():
    L = tb.lib()
    host = np.zeros(1 << 16, dtype=np.uint8)
    ws = tb.new_workspace(1 << 16)
    hp = ctypes.c_void_p(((host.ctypes.data + 255) // 256) * 256)
    rc = L.bitlinear_quant_act(hp, 0, 1, 256, ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                               None, None)
    assert rc == tb.BL_ERR_INVALID_ARG and "not device-accessible" in tb.last_error()


def test_misaligned_pointer_is_rejected():
    x = torch.zeros(4 * 256 + 16, dtype=torch.float32, device="cuda")
    xq = torch.zeros(4 * 256 + 16, dtype=torch.int8, device="cuda")
    s = torch.zeros(8, dtype=torch.float32, device="cuda")
    L = tb.lib()
    rc = L.bitlinear_quant_act(ctypes.c_void_p(x.data_ptr() + 4), 0, 4, 256, ctypes.c_void_p(xq.data_ptr()),
                               ctypes.c_void_p(s.data_ptr()), None, None)
    assert rc == tb.BL_ERR_MISALIGNED


def test_short_workspace_is_rejected():
    packed, gamma = tb.pack_weights(dev(weights(64, 256, seed=1)))
    x, _ = activations(4, 256, seed=2, dtype="f32")
    ws = tb.new_workspace(256)
    with pytest.raises(tb.BitLinearError) as e:
        tb.forward(packed, gamma, x, workspace=ws)
    assert e.value.code == tb.BL_ERR_WORKSPACE_TOO_SMALL


def test_forced_gemv_rejects_large_m():
    packed, gamma = tb.pack_weights(dev(weights(64, 256, seed=1)))
    x, _ = activations(17, 256, seed=2, dtype="f32")
    tb.set_path(tb.PATH_GEMV)
    try:
        with pytest.raises(tb.BitLinearError) as e:
            tb.forward(packed, gamma, x)
        assert e.value.code == tb.BL_ERR_UNSUPPORTED_SHAPE
    finally:
        tb.set_path(tb.PATH_AUTO)


def test_device_wait_times_out_and_context_survives():
    ws = tb.new_workspace(1 << 16)
    assert tb.device_status(ws) == tb.BL_OK
    tb.selftest_wait_timeout(ws, limit_us=2000)
    assert tb.device_status(ws) == tb.BL_ERR_DEVICE_TIMEOUT
    assert "ran out of time" in tb.last_error()
    assert tb.device_status(ws) == tb.BL_OK  # cleared
    # the context still runs real work
    packed, gamma = tb.pack_weights(dev(weights(128, 256, seed=3)))
    x, _ = activations(2, 256, seed=4, dtype="f32")
    y = tb.forward(packed, gamma, x, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()


@pytest.mark.parametrize("M", [1, 9, 40])
def test_no_writes_outside_outputs(M):
    N, K = 333, 320
    packed, gamma = tb.pack_weights(dev(weights(N, K, seed=M)))
    x, _ = activations(M, K, seed=M + 1, dtype="bf16")
    pad = 4096
    canary = 0x5A
    ybuf = torch.full((pad + M * N * 2 + pad,), canary, dtype=torch.uint8, device="cuda")
    abuf = torch.full((pad + M * N * 4 + pad,), canary, dtype=torch.uint8, device="cuda")
    y = ybuf[pad:pad + M * N * 2].view(torch.bfloat16).view(M, N)
    acc = abuf[pad:pad + M * N * 4].view(torch.int32).view(M, N)
    ws_bytes = tb.workspace_bytes(M, N, K)
    wbuf = torch.full((ws_bytes + pad,), canary, dtype=torch.uint8, device="cuda")
    wbuf[:256] = 0  # the status word starts at zero
    ws = wbuf[:ws_bytes]
    tb.forward(packed, gamma, x, y=y, acc_out=acc, workspace=ws)
    torch.cuda.synchronize()
    for buf in (ybuf[:pad], ybuf[-pad:], abuf[:pad], abuf[-pad:], wbuf[ws_bytes:]):
        assert (buf == canary).all()
    assert tb.device_status(ws) == tb.BL_OK


def test_default_argument_calls_launch_only_library_kernels():
    """A forward or chain call without a workspace uses the cached one: after the
    first call, the calls launch the library's kernels and nothing else (no
    allocation, no fill)."""
    from torch.profiler import ProfilerActivity, profile

    packed, gamma = tb.pack_weights(dev(weights(640, 1024, seed=5)))
    x, _ = activations(4, 1024, seed=6, dtype="bf16")
    y = torch.empty((4, 640), dtype=torch.bfloat16, device="cuda")
    layers = [tb.Layer(packed, gamma, x, torch.empty((4, 640), dtype=torch.bfloat16, device="cuda"))]
    tb.forward(packed, gamma, x, y=y)
    tb.layer_chain(layers)
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for _ in range(3):
            tb.forward(packed, gamma, x, y=y)
            tb.layer_chain(layers)
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    kernels = [n for n in names if "memcpy" not in n.lower() and "memset" not in n.lower()]
    assert kernels, "no kernel was recorded"
    assert all(n.startswith("void bl::") or n.startswith("bl::") for n in kernels), sorted(set(kernels))
