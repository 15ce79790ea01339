"""CPU oracle for the BitLinear W1.58A8 forward (numpy front end of ``bitlinear_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg are its only callers.  The ``ternary_weight_a8_b200``
package never imports it, and it imports nothing from that package.

Each function below is a thin wrapper of one C function; the C file's header
cites the passages of the BitNet b1.58 pages each step follows and lists the
readings taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import fcntl
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitlinear_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc if it is missing or stale."""
    with open(_SO + ".lock", "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
            tmp = _SO + ".tmp.%d" % os.getpid()
            subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
            os.replace(tmp, _SO)
    return _SO


_handle = None


def _lib():
    global _handle
    if _handle is None:
        # A mutation test may point this at a deliberately broken build.
        override = os.environ.get("BITLINEAR_ORACLE_LIB")
        lib = ctypes.CDLL(override if override else build())
        i64, vp = ctypes.c_int64, ctypes.c_void_p
        lib.oracle_absmean_gamma.argtypes = [vp, i64, i64, vp]
        lib.oracle_absmean_gamma.restype = ctypes.c_float
        lib.oracle_ternarize.argtypes = [vp, i64, ctypes.c_float, vp]
        lib.oracle_ternarize.restype = None
        lib.oracle_pack.argtypes = [vp, i64, i64, vp]
        lib.oracle_pack.restype = ctypes.c_int
        lib.oracle_unpack.argtypes = [vp, i64, i64, vp]
        lib.oracle_unpack.restype = ctypes.c_int
        lib.oracle_quant_act.argtypes = [vp, i64, i64, vp, vp, vp]
        lib.oracle_quant_act.restype = None
        lib.oracle_accumulate.argtypes = [vp, vp, i64, i64, i64, vp]
        lib.oracle_accumulate.restype = ctypes.c_int
        lib.oracle_dequant.argtypes = [vp, ctypes.c_float, vp, i64, i64, vp]
        lib.oracle_dequant.restype = None
        lib.oracle_round_f32.argtypes = [vp, i64, vp]
        lib.oracle_round_f32.restype = None
        lib.oracle_round_bf16.argtypes = [vp, i64, vp]
        lib.oracle_round_bf16.restype = None
        lib.oracle_rmsnorm.argtypes = [vp, i64, i64, vp, ctypes.c_float, ctypes.c_int, vp]
        lib.oracle_rmsnorm.restype = None
        lib.oracle_glu.argtypes = [vp, vp, i64, ctypes.c_int, ctypes.c_int, vp]
        lib.oracle_glu.restype = None
        lib.oracle_ste_grad_input.argtypes = [vp, vp, ctypes.c_float, i64, i64, i64, vp]
        lib.oracle_ste_grad_input.restype = None
        lib.oracle_ste_xhat.argtypes = [vp, vp, i64, i64, vp]
        lib.oracle_ste_xhat.restype = None
        lib.oracle_ste_grad_weight.argtypes = [vp, vp, i64, i64, i64, vp]
        lib.oracle_ste_grad_weight.restype = None
        _handle = lib
    return _handle


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def absmean_gamma(W: np.ndarray) -> tuple[np.float32, float]:
    """gamma = mean|W| (fp32) and the double sum it came from."""
    W = _c(W, np.float32)
    N, K = W.shape
    total = ctypes.c_double(0.0)
    g = _lib().oracle_absmean_gamma(W.ctypes.data, N, K, ctypes.byref(total))
    return np.float32(g), total.value


def ternarize(W: np.ndarray, gamma) -> np.ndarray:
    """t = clamp(round(W / (gamma + 1e-5)), -1, 1) as int8, same shape as W."""
    W = _c(W, np.float32)
    T = np.empty(W.shape, dtype=np.int8)
    _lib().oracle_ternarize(W.ctypes.data, W.size, float(np.float32(gamma)), T.ctypes.data)
    return T


def pack(T: np.ndarray) -> np.ndarray:
    """Ternary int8 ``[N][K]`` -> packed uint8 ``[N][K/4]`` (K % 16 == 0)."""
    T = _c(T, np.int8)
    N, K = T.shape
    P = np.empty((N, K // 4), dtype=np.uint8)
    rc = _lib().oracle_pack(T.ctypes.data, N, K, P.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_pack failed (%d)" % rc)
    return P


def unpack(P: np.ndarray, K: int) -> tuple[np.ndarray, bool]:
    """Packed ``[N][K/4]`` -> (ternary int8 ``[N][K]``, every code was 0..2)."""
    P = _c(P, np.uint8)
    N = P.shape[0]
    T = np.empty((N, K), dtype=np.int8)
    rc = _lib().oracle_unpack(P.ctypes.data, N, K, T.ctypes.data)
    if rc == -2:
        raise ValueError("K must be a multiple of 16")
    return T, rc == 0


def quant_act(x: np.ndarray):
    """Per-token absmax int8: returns (q int8 ``[M][K]``, s fp32 ``[M]``, rowsum int32 ``[M]``)."""
    x = _c(x, np.float32)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    r = np.empty(M, dtype=np.int32)
    _lib().oracle_quant_act(x.ctypes.data, M, K, q.ctypes.data, s.ctypes.data, r.ctypes.data)
    return q, s, r


def accumulate(q: np.ndarray, T: np.ndarray) -> np.ndarray:
    """acc[m][n] = sum_k q[m][k] * T[n][k] (int32; raises if a sum overflows)."""
    q = _c(q, np.int8)
    T = _c(T, np.int8)
    M, K = q.shape
    N = T.shape[0]
    assert T.shape[1] == K
    acc = np.empty((M, N), dtype=np.int32)
    rc = _lib().oracle_accumulate(q.ctypes.data, T.ctypes.data, M, N, K, acc.ctypes.data)
    if rc != 0:
        raise OverflowError("accumulator outside int32")
    return acc


def dequant(acc: np.ndarray, gamma, s: np.ndarray) -> np.ndarray:
    """y = acc * gamma / s[m] in double, ``[M][N]``."""
    acc = _c(acc, np.int32)
    s = _c(s, np.float32)
    M, N = acc.shape
    y = np.empty((M, N), dtype=np.float64)
    _lib().oracle_dequant(acc.ctypes.data, float(np.float32(gamma)), s.ctypes.data, M, N, y.ctypes.data)
    return y


def round_f32(y: np.ndarray) -> np.ndarray:
    y = _c(y, np.float64)
    out = np.empty(y.shape, dtype=np.float32)
    _lib().oracle_round_f32(y.ctypes.data, y.size, out.ctypes.data)
    return out


def round_bf16(y: np.ndarray) -> np.ndarray:
    """double -> bf16 bit patterns (uint16), one round-to-nearest-even."""
    y = _c(y, np.float64)
    out = np.empty(y.shape, dtype=np.uint16)
    _lib().oracle_round_bf16(y.ctypes.data, y.size, out.ctypes.data)
    return out


def pack_weights(W: np.ndarray):
    """The offline weight path: (packed ``[N][K/4]``, gamma, ternary ``[N][K]``)."""
    gamma, _ = absmean_gamma(W)
    T = ternarize(W, gamma)
    return pack(T), gamma, T


def forward(T: np.ndarray, gamma, x: np.ndarray):
    """The forward on ternary weights: returns (acc int32, y double, q, s, rowsum)."""
    q, s, r = quant_act(x)
    acc = accumulate(q, T)
    return acc, dequant(acc, gamma, s), q, s, r


def rmsnorm(x: np.ndarray, gain: np.ndarray | None, eps: float, out_bf16: bool) -> np.ndarray:
    """Per-token RMSNorm ``[M][K]`` -> fp32 values, rounded to bf16 when ``out_bf16``."""
    x = _c(x, np.float32)
    M, K = x.shape
    g = None if gain is None else _c(gain, np.float32)
    out = np.empty((M, K), dtype=np.float32)
    _lib().oracle_rmsnorm(x.ctypes.data, M, K, None if g is None else g.ctypes.data, float(np.float32(eps)),
                          1 if out_bf16 else 0, out.ctypes.data)
    return out


def rmsnorm_quant(x: np.ndarray, gain: np.ndarray | None, eps: float, out_bf16: bool):
    """The fused pre-norm: RMSNorm then per-token quantisation; returns (v, q, s, rowsum)."""
    v = rmsnorm(x, gain, eps, out_bf16)
    q, s, r = quant_act(v)
    return v, q, s, r


GLU_RELU2, GLU_SILU = 0, 1


def glu(gate: np.ndarray, up: np.ndarray, act: int, out_bf16: bool) -> np.ndarray:
    """h = act(gate) * up (act GLU_RELU2 or GLU_SILU), rounded to bf16 when ``out_bf16``."""
    gate = _c(gate, np.float32)
    up = _c(up, np.float32)
    assert gate.shape == up.shape
    out = np.empty(gate.shape, dtype=np.float32)
    _lib().oracle_glu(gate.ctypes.data, up.ctypes.data, gate.size, int(act), 1 if out_bf16 else 0, out.ctypes.data)
    return out


def glu_quant(gate: np.ndarray, up: np.ndarray, act: int, out_bf16: bool):
    """The FFN's gated activation then per-token quantisation; returns (h, q, s, rowsum)."""
    h = glu(gate, up, act, out_bf16)
    q, s, r = quant_act(h)
    return h, q, s, r


def ste_grad_input(dy: np.ndarray, T: np.ndarray, gamma) -> np.ndarray:
    """Straight-through dx = gamma * (dy . t), double ``[M][K]``."""
    dy = _c(dy, np.float32)
    T = _c(T, np.int8)
    M, N = dy.shape
    K = T.shape[1]
    assert T.shape[0] == N
    dx = np.empty((M, K), dtype=np.float64)
    _lib().oracle_ste_grad_input(dy.ctypes.data, T.ctypes.data, float(np.float32(gamma)), M, N, K, dx.ctypes.data)
    return dx


def ste_xhat(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """The stored dequantised activations bf16(q / s), as fp32 values ``[M][K]``."""
    q = _c(q, np.int8)
    s = _c(s, np.float32)
    M, K = q.shape
    out = np.empty((M, K), dtype=np.float32)
    _lib().oracle_ste_xhat(q.ctypes.data, s.ctypes.data, M, K, out.ctypes.data)
    return out


def ste_grad_weight(dy: np.ndarray, xhat: np.ndarray) -> np.ndarray:
    """Straight-through dW = dy^T . xhat, double ``[N][K]``."""
    dy = _c(dy, np.float32)
    xhat = _c(xhat, np.float32)
    M, N = dy.shape
    K = xhat.shape[1]
    assert xhat.shape[0] == M
    dw = np.empty((N, K), dtype=np.float64)
    _lib().oracle_ste_grad_weight(dy.ctypes.data, xhat.ctypes.data, M, N, K, dw.ctypes.data)
    return dw
