"""Seeded synthetic inputs for the BitLinear W1.58A8 forward.

Holds no BitLinear arithmetic: it only draws the latent weights and the
activations that the oracle tests and the CUDA path both consume (see
``synth.c`` for the generator's definition).  The shapes and distributions
follow the workloads of the ternary-weight pages: latent weights
N(0, 0.02) in nn.Linear layout ``[N][K]``; activations N(0, 1), with 1 % of
the channels (chosen by a seeded Fisher-Yates shuffle) scaled by 20 before
the bf16 rounding, as outlier channels.
"""
from __future__ import annotations

import ctypes
import fcntl
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_SO = os.path.join(_HERE, "libsynth.so")

WEIGHT_STD = 0.02
OUTLIER_FRACTION = 0.01
OUTLIER_SCALE = 20.0


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` with gcc (OpenMP) if it is missing or stale."""
    lock_path = _SO + ".lock"
    with open(lock_path, "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
            tmp = _SO + ".tmp.%d" % os.getpid()
            subprocess.check_call(
                ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
            )
            os.replace(tmp, _SO)
    return _SO


_lib_handle = None


def _lib():
    global _lib_handle
    if _lib_handle is None:
        lib = ctypes.CDLL(build())
        u64, i64, i32, f64 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        vp = ctypes.c_void_p
        lib.synth_normal_f32.argtypes = [u64, u64, u64, i64, f64, f64, vp]
        lib.synth_normal_f32.restype = None
        lib.synth_choose_channels.argtypes = [u64, u64, i32, i32, vp]
        lib.synth_choose_channels.restype = ctypes.c_int
        lib.synth_activations_f32.argtypes = [u64, u64, i64, i64, vp, f64, vp]
        lib.synth_activations_f32.restype = None
        lib.synth_f32_to_bf16.argtypes = [vp, i64, vp]
        lib.synth_f32_to_bf16.restype = None
        lib.synth_bf16_to_f32.argtypes = [vp, i64, vp]
        lib.synth_bf16_to_f32.restype = None
        _lib_handle = lib
    return _lib_handle


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def normal_f32(n: int, seed: int, stream: int = 0, mean: float = 0.0, std: float = 1.0,
               offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _lib().synth_normal_f32(seed, stream, offset, n, mean, std, _ptr(out))
    return out


def latent_weights(N: int, K: int, seed: int, stream: int = 1, std: float = WEIGHT_STD) -> np.ndarray:
    """Latent (shadow) weights, fp32 ``[N][K]`` ~ N(0, std)."""
    return normal_f32(N * K, seed, stream, 0.0, std).reshape(N, K)


def outlier_count(K: int, fraction: float = OUTLIER_FRACTION) -> int:
    return int(round(fraction * K))


def outlier_channels(K: int, seed: int, stream: int = 3, fraction: float = OUTLIER_FRACTION) -> np.ndarray:
    """``round(fraction*K)`` distinct channel indices from a seeded shuffle."""
    count = outlier_count(K, fraction)
    scratch = np.empty(max(K, 1), dtype=np.int32)
    rc = _lib().synth_choose_channels(seed, stream, K, count, _ptr(scratch))
    if rc != 0:
        raise ValueError("bad outlier count")
    return scratch[:count].copy()


def activations_f32(M: int, K: int, seed: int, stream: int = 2, outliers: bool = True,
                    outlier_seed: int | None = None) -> np.ndarray:
    """fp32 activations ``[M][K]`` ~ N(0, 1), outlier channels scaled by 20."""
    out = np.empty((M, K), dtype=np.float32)
    mask = None
    if outliers:
        mask = np.zeros(K, dtype=np.uint8)
        mask[outlier_channels(K, seed if outlier_seed is None else outlier_seed)] = 1
    _lib().synth_activations_f32(seed, stream, M, K, _ptr(mask) if mask is not None else None,
                                 OUTLIER_SCALE, _ptr(out))
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _lib().synth_f32_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.float32)
    _lib().synth_bf16_to_f32(_ptr(b), b.size, _ptr(out))
    return out


def activations_bf16(M: int, K: int, seed: int, stream: int = 2, outliers: bool = True):
    """bf16 activations: returns (bits uint16 ``[M][K]``, exact fp32 values)."""
    bits = f32_to_bf16_bits(activations_f32(M, K, seed, stream, outliers))
    return bits, bf16_bits_to_f32(bits)


# Workloads of the ternary-weight pages, as (name, layers, token counts, dtype).
# A layer is (K in, N out); the 70B-class chain runs QKV, O, gate, up, down,
# gate and up sharing one input.
CHAIN_70B = [(8192, 10240), (8192, 8192), (8192, 28672), (8192, 28672), (28672, 8192)]
CHAIN_70B_SHARED_INPUT = [False, False, False, True, False]

WORKLOADS = {
    "single_256": dict(layers=[(256, 256)], tokens=[4], dtype="f32"),
    "decode_2b": dict(layers=[(2560, 6912), (2560, 2560)], tokens=[1], dtype="bf16"),
    "decode_3b": dict(layers=[(3200, 8640), (8640, 3200)], tokens=[1, 2, 4, 8, 16], dtype="bf16"),
    "prefill_2b": dict(layers=[(2560, 6912)], tokens=[2048], dtype="bf16"),
    "chain_70b": dict(layers=CHAIN_70B, tokens=[1, 8], dtype="bf16"),
}
