"""B200-native BitLinear W1.58A8 forward (BitNet b1.58), Python binding.

A thin ctypes binding of ``libbitlinear.so``, whose C ABI is declared in
``include/bitlinear.h``.  This module only marshals arguments: PyTorch
provides device memory and the current stream; every step of the forward
runs in the library's CUDA kernels.  There is no CPU fallback: if the
library is missing or no GPU is present, the calls raise.

Calls (same names as the C ABI, without the ``bitlinear_`` prefix):
``pack_weights``, ``quant_act``, ``forward``, ``forward_quantized``,
``layer_chain``, ``device_status``, plus workspace helpers.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbitlinear.so")

BL_F32, BL_BF16 = 0, 1
BL_OK = 0
BL_ERR_INVALID_ARG = -1
BL_ERR_UNSUPPORTED_SHAPE = -2
BL_ERR_MISALIGNED = -3
BL_ERR_WORKSPACE_TOO_SMALL = -4
BL_ERR_CUDA = -5
BL_ERR_DEVICE_TIMEOUT = -6

PATH_AUTO, PATH_GEMV, PATH_GEMM = 0, 1, 2


class BitLinearError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__("bitlinear error %d: %s" % (code, message))
        self.code = code


class bl_layer(ctypes.Structure):
    _fields_ = [
        ("packed", ctypes.c_void_p),
        ("gamma", ctypes.c_void_p),
        ("N", ctypes.c_int),
        ("K", ctypes.c_int),
        ("x", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("xq", ctypes.c_void_p),
        ("scale", ctypes.c_void_p),
        ("rowsum", ctypes.c_void_p),
        ("acc_out", ctypes.c_void_p),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libbitlinear.so is not built; run `python -m ternary_weight_a8_b200._build` "
                "(or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        sigs = {
            "bitlinear_pack_workspace_bytes": (sz, [i32, i32]),
            "bitlinear_pack_weights": (i32, [vp, i32, i32, vp, vp, vp, sz, vp]),
            "bitlinear_quant_act": (i32, [vp, i32, i32, i32, vp, vp, vp, vp]),
            "bitlinear_rmsnorm_quant": (i32, [vp, i32, i32, i32, vp, ctypes.c_float, vp, vp, vp, vp, vp]),
            "bitlinear_glu_quant": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]),
            "bitlinear_gate_up_glu_workspace_bytes": (sz, [i32, i32, i32]),
            "bitlinear_gate_up_glu": (i32, [vp, vp, vp, vp, i32, i32, vp, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp]),
            "bitlinear_forward_lut": (i32, [vp, vp, i32, i32, vp, vp, vp, i32, vp, i32, vp, vp]),
            "bitlinear_ste_workspace_bytes": (sz, [i32, i32, i32]),
            "bitlinear_ste_backward": (i32, [vp, vp, i32, i32, vp, vp, vp, i32, vp, i32, vp, vp, sz, vp]),
            "bitlinear_workspace_bytes": (sz, [i32, i32, i32]),
            "bitlinear_forward": (i32, [vp, vp, i32, i32, vp, i32, i32, vp, i32, vp, vp, sz, vp]),
            "bitlinear_forward_quantized": (i32, [vp, vp, i32, i32, vp, vp, vp, i32, vp, i32, vp, vp, sz, vp]),
            "bitlinear_chain_workspace_bytes": (sz, [ctypes.POINTER(bl_layer), i32, i32]),
            "bitlinear_layer_chain": (i32, [ctypes.POINTER(bl_layer), i32, i32, i32, i32, vp, sz, vp]),
            "bitlinear_device_status": (i32, [vp, vp]),
            "bitlinear_selftest_wait_timeout": (i32, [vp, sz, i32, vp]),
            "bitlinear_set_path": (i32, [i32]),
            "bitlinear_set_decode_split": (i32, [i32]),
            "bitlinear_set_decode_form": (i32, [i32]),
            "bitlinear_forward_noalloc": (i32, [vp, vp, i32, i32, vp, i32, i32, vp, i32, vp, vp]),
            "bitlinear_noalloc_status": (i32, [vp]),
            "bitlinear_last_error": (ctypes.c_char_p, []),
            "bitlinear_version": (i32, []),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def last_error() -> str:
    return lib().bitlinear_last_error().decode()


def _check(rc: int) -> None:
    if rc != BL_OK:
        raise BitLinearError(rc, last_error())


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return BL_F32
    if dt == torch.bfloat16:
        return BL_BF16
    raise ValueError("unsupported dtype %s (float32 or bfloat16)" % dt)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: torch.cuda.Stream | None = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def set_path(path: int) -> None:
    """Force the product kernel on this thread: PATH_AUTO, PATH_GEMV or PATH_GEMM."""
    _check(lib().bitlinear_set_path(path))


def set_decode_split(ctas: int) -> None:
    """Force the decode kernel's K-split to ``ctas`` CTAs per unit on this thread (0: automatic)."""
    _check(lib().bitlinear_set_decode_split(int(ctas)))


DECODE_FORM_AUTO, DECODE_FORM_CUDA_CORES, DECODE_FORM_TENSOR_CORES = 0, 1, 2


def set_decode_form(form: int) -> None:
    """Force the decode product's form for 9-16 tokens on this thread (DECODE_FORM_*)."""
    _check(lib().bitlinear_set_decode_form(int(form)))


def version() -> int:
    return lib().bitlinear_version()


# ----------------------------------------------------------------------------
# Workspaces
# ----------------------------------------------------------------------------

def pack_workspace_bytes(N: int, K: int) -> int:
    return lib().bitlinear_pack_workspace_bytes(N, K)


def workspace_bytes(M: int, N: int, K: int) -> int:
    return lib().bitlinear_workspace_bytes(M, N, K)


def new_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zeroed uint8 device buffer of at least ``nbytes`` (the status word starts at zero)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


_WS_CACHE: dict = {}


def cached_workspace(nbytes: int, device=None, stream=None) -> torch.Tensor:
    """The workspace a call without an explicit one uses: one zeroed buffer per
    (device, stream), kept between calls and replaced by a larger one only
    when a call needs more.  Calls on one stream are ordered, so they may share
    it; the library leaves its zeroed parts zeroed."""
    dev = torch.device(device if device is not None else "cuda")
    if dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    key = (dev.index, s.cuda_stream)
    ws = _WS_CACHE.get(key)
    if ws is None or ws.numel() < nbytes:
        with torch.cuda.stream(s):
            ws = new_workspace(nbytes, dev)
        _WS_CACHE[key] = ws
    return ws


# ----------------------------------------------------------------------------
# Calls
# ----------------------------------------------------------------------------

def pack_weights(W: torch.Tensor, packed: torch.Tensor | None = None, gamma: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None, stream=None):
    """Latent fp32 weights ``[N][K]`` -> (packed uint8 ``[N][K/4]``, gamma fp32 ``[1]``)."""
    N, K = W.shape
    if packed is None:
        packed = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    if workspace is None:
        workspace = cached_workspace(pack_workspace_bytes(N, K), W.device, stream)
    _check(lib().bitlinear_pack_weights(_ptr(W), N, K, _ptr(packed), _ptr(gamma), _ptr(workspace),
                                        workspace.numel(), _stream(stream)))
    return packed, gamma


def quant_act(x: torch.Tensor, xq=None, scale=None, rowsum=None, stream=None):
    """Activations ``[M][K]`` (fp32/bf16) -> (int8 q ``[M][K]``, fp32 s ``[M]``, int32 rowsum ``[M]``)."""
    M, K = x.shape
    dev = x.device
    xq = torch.empty((M, K), dtype=torch.int8, device=dev) if xq is None else xq
    scale = torch.empty(M, dtype=torch.float32, device=dev) if scale is None else scale
    rowsum = torch.empty(M, dtype=torch.int32, device=dev) if rowsum is None else rowsum
    _check(lib().bitlinear_quant_act(_ptr(x), _dtype_code(x.dtype), M, K, _ptr(xq), _ptr(scale),
                                     _ptr(rowsum), _stream(stream)))
    return xq, scale, rowsum


def rmsnorm_quant(x: torch.Tensor, gain: torch.Tensor | None = None, eps: float = 1e-6, x_norm=None, xq=None,
                  scale=None, rowsum=None, stream=None):
    """RMSNorm fused with the per-token quantisation: returns (xq, scale, rowsum), and also
    the normalised activations first when ``x_norm`` is True or a tensor."""
    M, K = x.shape
    dev = x.device
    xq = torch.empty((M, K), dtype=torch.int8, device=dev) if xq is None else xq
    scale = torch.empty(M, dtype=torch.float32, device=dev) if scale is None else scale
    rowsum = torch.empty(M, dtype=torch.int32, device=dev) if rowsum is None else rowsum
    norm = torch.empty_like(x) if x_norm is True else (x_norm if isinstance(x_norm, torch.Tensor) else None)
    _check(lib().bitlinear_rmsnorm_quant(_ptr(x), _dtype_code(x.dtype), M, K, _ptr(gain), float(eps), _ptr(norm),
                                         _ptr(xq), _ptr(scale), _ptr(rowsum), _stream(stream)))
    return (norm, xq, scale, rowsum) if norm is not None else (xq, scale, rowsum)


def forward_lut(packed: torch.Tensor, gamma: torch.Tensor, xq: torch.Tensor, scale: torch.Tensor,
                rowsum: torch.Tensor, out_dtype=torch.bfloat16, y: torch.Tensor | None = None,
                acc_out: torch.Tensor | bool | None = None, stream=None):
    """One token's product by table lookup (the T-MAC-style decode), on codes from ``quant_act``."""
    N = packed.shape[0]
    M, K = xq.shape
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=xq.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=xq.device) if acc_out is True else (
        acc_out if isinstance(acc_out, torch.Tensor) else None)
    _check(lib().bitlinear_forward_lut(_ptr(packed), _ptr(gamma), N, K, _ptr(xq), _ptr(scale), _ptr(rowsum), M,
                                       _ptr(y), _dtype_code(y.dtype), _ptr(acc), _stream(stream)))
    return (y, acc) if acc is not None else y


def ste_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().bitlinear_ste_workspace_bytes(M, N, K))


def ste_backward(packed: torch.Tensor, gamma: torch.Tensor, K: int, dy: torch.Tensor, xq: torch.Tensor,
                 scale: torch.Tensor, dx=True, dx_dtype=torch.float32, dw=True, workspace=None, stream=None):
    """The straight-through backward: returns (dx [M][K] or None, dW [N][K] fp32 or None)."""
    M, N = dy.shape
    if dy.dtype != torch.bfloat16:
        raise ValueError("dy must be bf16")
    dev = dy.device
    dxt = torch.empty((M, K), dtype=dx_dtype, device=dev) if dx is True else (dx if isinstance(dx, torch.Tensor) else None)
    dwt = torch.empty((N, K), dtype=torch.float32, device=dev) if dw is True else (dw if isinstance(dw, torch.Tensor) else None)
    if workspace is None:
        workspace = cached_workspace(ste_workspace_bytes(M, N, K), dev, stream)
    _check(lib().bitlinear_ste_backward(_ptr(packed), _ptr(gamma), N, K, _ptr(dy), _ptr(xq), _ptr(scale), M, _ptr(dxt),
                                        _dtype_code(dxt.dtype) if dxt is not None else 0, _ptr(dwt), _ptr(workspace),
                                        workspace.numel(), _stream(stream)))
    return dxt, dwt


GLU_RELU2, GLU_SILU = 0, 1


def glu_quant(gate: torch.Tensor, up: torch.Tensor, act: int = GLU_RELU2, h=None, xq=None, scale=None, rowsum=None,
              stream=None):
    """h = act(gate) * up fused with its per-token quantisation (the down BitLinear's input):
    returns (xq, scale, rowsum), and h first when ``h`` is True or a tensor."""
    if gate.shape != up.shape or gate.dtype != up.dtype:
        raise ValueError("gate and up must have the same shape and dtype")
    M, N = gate.shape
    dev = gate.device
    xq = torch.empty((M, N), dtype=torch.int8, device=dev) if xq is None else xq
    scale = torch.empty(M, dtype=torch.float32, device=dev) if scale is None else scale
    rowsum = torch.empty(M, dtype=torch.int32, device=dev) if rowsum is None else rowsum
    hout = torch.empty_like(gate) if h is True else (h if isinstance(h, torch.Tensor) else None)
    _check(lib().bitlinear_glu_quant(_ptr(gate), _ptr(up), _dtype_code(gate.dtype), M, N, int(act), _ptr(hout),
                                     _ptr(xq), _ptr(scale), _ptr(rowsum), _stream(stream)))
    return (hout, xq, scale, rowsum) if hout is not None else (xq, scale, rowsum)


def gate_up_glu_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().bitlinear_gate_up_glu_workspace_bytes(M, N, K))


def gate_up_glu(packed_gate: torch.Tensor, gamma_gate: torch.Tensor, packed_up: torch.Tensor,
                gamma_up: torch.Tensor, x: torch.Tensor, act: int = GLU_RELU2, h=None, xq=None, scale=None,
                rowsum=None, workspace=None, stream=None):
    """The FFN's gate and up BitLinears, h = act(gate) * up and h's quantisation for the down
    BitLinear in one call: returns (xq, scale, rowsum), and h first when ``h`` is True or a tensor."""
    N = packed_gate.shape[0]
    M, K = x.shape
    dev = x.device
    xq = torch.empty((M, N), dtype=torch.int8, device=dev) if xq is None else xq
    scale = torch.empty(M, dtype=torch.float32, device=dev) if scale is None else scale
    rowsum = torch.empty(M, dtype=torch.int32, device=dev) if rowsum is None else rowsum
    hout = torch.empty((M, N), dtype=x.dtype, device=dev) if h is True else (h if isinstance(h, torch.Tensor) else None)
    if workspace is None:
        workspace = cached_workspace(gate_up_glu_workspace_bytes(M, N, K), dev, stream)
    _check(lib().bitlinear_gate_up_glu(_ptr(packed_gate), _ptr(gamma_gate), _ptr(packed_up), _ptr(gamma_up), N, K,
                                       _ptr(x), _dtype_code(x.dtype), M, int(act), _ptr(hout), _ptr(xq), _ptr(scale),
                                       _ptr(rowsum), _ptr(workspace), workspace.numel(), _stream(stream)))
    return (hout, xq, scale, rowsum) if hout is not None else (xq, scale, rowsum)


def forward(packed: torch.Tensor, gamma: torch.Tensor, x: torch.Tensor, out_dtype=torch.bfloat16,
            y: torch.Tensor | None = None, acc_out: torch.Tensor | bool | None = None,
            workspace: torch.Tensor | None = None, stream=None):
    """y = BitLinear(x): returns y, or (y, acc) when ``acc_out`` is True or a tensor."""
    N = packed.shape[0]
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=x.device)
    acc = None
    if acc_out is True:
        acc = torch.empty((M, N), dtype=torch.int32, device=x.device)
    elif isinstance(acc_out, torch.Tensor):
        acc = acc_out
    if workspace is None:
        workspace = cached_workspace(workspace_bytes(M, N, K), x.device, stream)
    _check(lib().bitlinear_forward(_ptr(packed), _ptr(gamma), N, K, _ptr(x), _dtype_code(x.dtype), M,
                                   _ptr(y), _dtype_code(y.dtype), _ptr(acc), _ptr(workspace),
                                   workspace.numel(), _stream(stream)))
    return (y, acc) if acc is not None else y


def forward_quantized(packed: torch.Tensor, gamma: torch.Tensor, xq: torch.Tensor, scale: torch.Tensor,
                      rowsum: torch.Tensor, out_dtype=torch.bfloat16, y: torch.Tensor | None = None,
                      acc_out: torch.Tensor | bool | None = None, workspace: torch.Tensor | None = None,
                      stream=None):
    """The product + dequantisation on activations from ``quant_act``."""
    N = packed.shape[0]
    M, K = xq.shape
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=xq.device)
    acc = None
    if acc_out is True:
        acc = torch.empty((M, N), dtype=torch.int32, device=xq.device)
    elif isinstance(acc_out, torch.Tensor):
        acc = acc_out
    if workspace is None:
        workspace = cached_workspace(workspace_bytes(M, N, K), xq.device, stream)
    _check(lib().bitlinear_forward_quantized(_ptr(packed), _ptr(gamma), N, K, _ptr(xq), _ptr(scale),
                                             _ptr(rowsum), M, _ptr(y), _dtype_code(y.dtype), _ptr(acc),
                                             _ptr(workspace), workspace.numel(), _stream(stream)))
    return (y, acc) if acc is not None else y


@dataclass
class Layer:
    """One BitLinear of a chain.  ``x`` is the input ``[M][K]``; or give
    ``xq``/``scale``/``rowsum`` (codes from ``quant_act`` or ``glu_quant``)
    instead, and ``x`` may be None.  ``acc_out`` (int32 ``[M][N]``) receives the
    exact accumulators when given."""
    packed: torch.Tensor
    gamma: torch.Tensor
    x: torch.Tensor | None
    y: torch.Tensor
    xq: torch.Tensor | None = None
    scale: torch.Tensor | None = None
    rowsum: torch.Tensor | None = None
    acc_out: torch.Tensor | None = None

    @property
    def tokens(self) -> int:
        return (self.x if self.x is not None else self.xq).shape[0]

    @property
    def K(self) -> int:
        return (self.x if self.x is not None else self.xq).shape[1]


def _layer_array(layers: Sequence[Layer]):
    arr = (bl_layer * len(layers))()
    for i, L in enumerate(layers):
        arr[i] = bl_layer(_ptr(L.packed), _ptr(L.gamma), L.packed.shape[0], L.K, _ptr(L.x), _ptr(L.y),
                          _ptr(L.xq), _ptr(L.scale), _ptr(L.rowsum), _ptr(L.acc_out))
    return arr


def chain_workspace_bytes(layers: Sequence[Layer], M: int) -> int:
    arr = _layer_array(layers)
    return lib().bitlinear_chain_workspace_bytes(arr, len(layers), M)


def layer_chain(layers: Sequence[Layer], workspace: torch.Tensor | None = None, stream=None) -> None:
    """Runs the layers back to back; each writes its ``y``.  Same-x neighbours share one quantisation."""
    if not layers:
        return
    M = layers[0].tokens
    arr = _layer_array(layers)
    if workspace is None:
        workspace = cached_workspace(lib().bitlinear_chain_workspace_bytes(arr, len(layers), M), layers[0].y.device,
                                     stream)
    x_dtype = next((L.x.dtype for L in layers if L.x is not None), layers[0].y.dtype)
    _check(lib().bitlinear_layer_chain(arr, len(layers), M, _dtype_code(x_dtype), _dtype_code(layers[0].y.dtype),
                                       _ptr(workspace), workspace.numel(), _stream(stream)))


class ChainPlan:
    """A ``layer_chain`` call marshalled once, for a loop that runs the same
    layers (same tensors) every step: ``run`` is then a single library call.
    The plan keeps references to the layers' tensors; it is invalid once one
    of them is replaced or freed."""

    def __init__(self, layers: Sequence[Layer], workspace: torch.Tensor | None = None, stream=None):
        if not layers:
            raise ValueError("a chain plan needs at least one layer")
        self.layers = list(layers)
        self.M = self.layers[0].tokens
        self._arr = _layer_array(self.layers)
        if workspace is None:
            workspace = new_workspace(lib().bitlinear_chain_workspace_bytes(self._arr, len(self.layers), self.M))
        self.workspace = workspace
        x_dtype = next((L.x.dtype for L in self.layers if L.x is not None), self.layers[0].y.dtype)
        self._args = (self._arr, len(self.layers), self.M, _dtype_code(x_dtype), _dtype_code(self.layers[0].y.dtype),
                      _ptr(workspace), workspace.numel())
        self._stream = _stream(stream) if stream is not None else None
        self._call = lib().bitlinear_layer_chain

    def run(self, stream=None) -> None:
        """The chain on ``stream`` (else the plan's stream, else the current stream)."""
        s = _stream(stream) if stream is not None else (self._stream or _stream(None))
        _check(self._call(*self._args, s))


def prepare_chain(layers: Sequence[Layer], workspace: torch.Tensor | None = None, stream=None) -> ChainPlan:
    """``layer_chain``'s arguments marshalled once (see ChainPlan)."""
    return ChainPlan(layers, workspace, stream)


def forward_noalloc(packed: torch.Tensor, gamma: torch.Tensor, x: torch.Tensor, y: torch.Tensor,
                    acc_out: torch.Tensor | None = None, stream=None) -> None:
    """The forward without a workspace (the library's fixed scratch): writes ``y`` (and ``acc_out``)."""
    N = packed.shape[0]
    M, K = x.shape
    _check(lib().bitlinear_forward_noalloc(_ptr(packed), _ptr(gamma), N, K, _ptr(x), _dtype_code(x.dtype), M, _ptr(y),
                                           _dtype_code(y.dtype), _ptr(acc_out), _stream(stream)))


def noalloc_status(stream=None) -> int:
    """Synchronises and returns BL_OK or BL_ERR_DEVICE_TIMEOUT for the no-allocation calls (clearing it)."""
    return lib().bitlinear_noalloc_status(_stream(stream))


def device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronises and returns BL_OK or BL_ERR_DEVICE_TIMEOUT (clearing the status word)."""
    return lib().bitlinear_device_status(_ptr(workspace), _stream(stream))


def selftest_wait_timeout(workspace: torch.Tensor, limit_us: int, stream=None) -> None:
    _check(lib().bitlinear_selftest_wait_timeout(_ptr(workspace), workspace.numel(), limit_us, _stream(stream)))
