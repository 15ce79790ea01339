"""Helpers shared by the GPU parity tests: moving seeded inputs to the device,
running the oracle on the same inputs, and the comparisons with their bars.

Bars (stated once, used everywhere):
  * packed weights, gamma, int8 activations, scales, row sums and int32
    accumulators: bit-exact;
  * fp32 outputs: |y - y_ref| <= 1e-6 * |y_ref|, and exactly 0 where acc == 0
    (the kernel computes fp32(acc) * fp32(gamma / s), two roundings, so its
    relative error is below 2**-23 ~= 1.2e-7);
  * bf16 outputs: within 1 bf16 ulp of the oracle's single rounding of the
    exact value.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

Y_F32_RTOL = 1e-6
Y_BF16_ULPS = 1


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32_bits(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def bf16_ordered(bits: np.ndarray) -> np.ndarray:
    """Map bf16 bit patterns to integers whose difference counts ulps."""
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)


def assert_y_matches(y: torch.Tensor, y_ref: np.ndarray, acc_ref: np.ndarray | None = None) -> None:
    """Check a device output against the oracle's double result at the stated bar."""
    if y.dtype == torch.float32:
        got = y.cpu().numpy().astype(np.float64)
        err = np.abs(got - y_ref)
        bad = err > Y_F32_RTOL * np.abs(y_ref)
        if acc_ref is not None:
            zero = acc_ref == 0
            bad |= zero & (got != 0)
        assert not bad.any(), "fp32 mismatch at %s: got %r want %r" % (
            np.argwhere(bad)[:5].tolist(), got[bad][:5], y_ref[bad][:5])
    elif y.dtype == torch.bfloat16:
        got = bf16_ordered(bf16_bits(y))
        want = bf16_ordered(oracle.round_bf16(y_ref))
        d = np.abs(got - want)
        assert d.max(initial=0) <= Y_BF16_ULPS, "bf16 off by %d ulps at %s" % (
            d.max(), np.argwhere(d > Y_BF16_ULPS)[:5].tolist())
    else:
        raise AssertionError(y.dtype)


def weights(N: int, K: int, seed: int, stream: int = 1) -> np.ndarray:
    return synth.latent_weights(N, K, seed=seed, stream=stream)


def activations(M: int, K: int, seed: int, dtype: str):
    """(device tensor, exact fp32 values as numpy) for fp32 or bf16 activations."""
    if dtype == "bf16":
        bits, xf = synth.activations_bf16(M, K, seed=seed)
        return bf16_dev(bits), xf
    xf = synth.activations_f32(M, K, seed=seed)
    return dev(xf), xf
