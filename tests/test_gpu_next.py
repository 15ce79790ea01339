"""GPU parity of the rows built beyond the forward itself, against the oracle.

Fused pre-norm: RMSNorm (gain optional) fused with the per-token
quantisation, compared with the oracle's RMSNorm followed by its
quantisation.  Gated activation: h = act(gate) * up fused with the
quantisation of the down BitLinear's input (bars below).  The normalised activations, codes, scales and code sums are
compared bit for bit (the norm's mean of squares is summed in double on both
sides, so its order changes only double's last bits and, in practice, never
the fp32 factor derived from it).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_weight_a8_b200 as tb
from parity import activations, assert_y_matches, bf16_bits, bf16_dev, bf16_ordered, dev, f32_bits, weights

pytestmark = pytest.mark.gpu


def _gain(K, seed):
    """A per-channel gain around 1 (what a trained norm weight looks like)."""
    return (1.0 + 0.1 * synth.activations_f32(1, K, seed=seed)[0]).astype(np.float32)


@pytest.mark.parametrize("M,K,dtype,with_gain,eps", [
    (1, 2560, "bf16", True, 1e-6), (4, 64, "f32", False, 1e-5), (16, 8640, "bf16", True, 1e-6),
    (2048, 2560, "bf16", True, 1e-6), (3, 28672, "bf16", False, 1e-6), (5, 8192, "f32", True, 0.0),
    (7, 32768 + 1024, "bf16", True, 1e-6),  # longer than a block holds in registers: read twice
])
def test_rmsnorm_quant_parity(M, K, dtype, with_gain, eps):
    x, xf = activations(M, K, seed=M * 3 + K, dtype=dtype)
    g = _gain(K, seed=K) if with_gain else None
    v_ref, q_ref, s_ref, r_ref = oracle.rmsnorm_quant(xf, g, eps, dtype == "bf16")
    v, q, s, r = tb.rmsnorm_quant(x, None if g is None else dev(g), eps=eps, x_norm=True)
    if dtype == "bf16":
        want = (f32_bits(v_ref) >> 16).astype(np.uint16)
        assert np.array_equal(bf16_bits(v), want)
    else:
        assert np.array_equal(f32_bits(v.cpu().numpy()), f32_bits(v_ref))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
    assert np.array_equal(r.cpu().numpy(), r_ref)


def test_rmsnorm_quant_degenerate_tokens():
    """A zero token, a one-hot token and a constant token."""
    K = 256
    xf = np.zeros((3, K), np.float32)
    xf[1, 17] = -3.0
    xf[2, :] = 0.5
    x = dev(xf)
    v_ref, q_ref, s_ref, r_ref = oracle.rmsnorm_quant(xf, None, 1e-6, False)
    v, q, s, r = tb.rmsnorm_quant(x, eps=1e-6, x_norm=True)
    assert np.array_equal(f32_bits(v.cpu().numpy()), f32_bits(v_ref))
    assert np.array_equal(q.cpu().numpy(), q_ref) and np.array_equal(r.cpu().numpy(), r_ref)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
    assert not q.cpu().numpy()[0].any()


def test_rmsnorm_codes_feed_the_product():
    """Normalised codes into the product: the same result as the oracle's norm, quantisation and product."""
    M, N, K = 3, 700, 2560
    W = weights(N, K, seed=11)
    packed_ref, gamma_ref, T = oracle.pack_weights(W)
    x, xf = activations(M, K, seed=12, dtype="bf16")
    g = _gain(K, seed=13)
    v_ref, q_ref, s_ref, r_ref = oracle.rmsnorm_quant(xf, g, 1e-6, True)
    acc_ref = oracle.accumulate(q_ref, T)
    y_ref = oracle.dequant(acc_ref, gamma_ref, s_ref)
    xq, s, r = tb.rmsnorm_quant(x, dev(g), eps=1e-6)
    y, acc = tb.forward_quantized(dev(packed_ref), dev(np.array([gamma_ref], np.float32)), xq, s, r,
                                  out_dtype=torch.bfloat16, acc_out=True)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_y_matches(y, y_ref, acc_ref)


def test_rmsnorm_rejects_bad_eps():
    x = torch.zeros((1, 64), dtype=torch.float32, device="cuda")
    for eps in (-1.0, float("inf"), float("nan")):
        with pytest.raises(tb.BitLinearError) as e:
            tb.rmsnorm_quant(x, eps=eps)
        assert e.value.code == tb.BL_ERR_INVALID_ARG


# ----------------------------------------------------------------------------
# The FFN's gated activation fused with the down BitLinear's quantisation.
# Squared ReLU is exact fp32 arithmetic: h, codes, scales and sums bit for
# bit.  SiLU calls the device expf (a few fp32 ulps from the exact value):
# h within 1 bf16 ulp (fp32: 8 ulps) of the oracle's one rounding of the
# exact value, and the codes exactly those of the oracle's quantisation of
# the kernel's own h (the integer decision taken on the same values).
# ----------------------------------------------------------------------------

def _gate_up(M, N, dtype, seed):
    g, gf = activations(M, N, seed=seed, dtype=dtype)
    u, uf = activations(M, N, seed=seed + 1, dtype=dtype)
    return g, gf, u, uf


@pytest.mark.parametrize("M,N,dtype", [(1, 6912, "bf16"), (16, 28672, "bf16"), (2048, 6912, "bf16"),
                                       (5, 640, "f32"), (3, 33792, "bf16")])
def test_glu_relu2_quant_parity(M, N, dtype):
    g, gf, u, uf = _gate_up(M, N, dtype, seed=N + M)
    h_ref, q_ref, s_ref, r_ref = oracle.glu_quant(gf, uf, oracle.GLU_RELU2, dtype == "bf16")
    h, q, s, r = tb.glu_quant(g, u, tb.GLU_RELU2, h=True)
    if dtype == "bf16":
        assert np.array_equal(bf16_bits(h), (f32_bits(h_ref) >> 16).astype(np.uint16))
    else:
        assert np.array_equal(f32_bits(h.cpu().numpy()), f32_bits(h_ref))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
    assert np.array_equal(r.cpu().numpy(), r_ref)


@pytest.mark.parametrize("M,N,dtype", [(1, 6912, "bf16"), (64, 2560, "bf16"), (4, 1024, "f32")])
def test_glu_silu_quant_parity(M, N, dtype):
    g, gf, u, uf = _gate_up(M, N, dtype, seed=N + 2 * M)
    h_ref = oracle.glu(gf, uf, oracle.GLU_SILU, dtype == "bf16")
    h, q, s, r = tb.glu_quant(g, u, tb.GLU_SILU, h=True)
    if dtype == "bf16":
        hv = (bf16_bits(h).astype(np.uint32) << 16).view(np.float32)
        d = np.abs(bf16_ordered(bf16_bits(h)) - bf16_ordered((f32_bits(h_ref) >> 16).astype(np.uint16)))
        assert d.max() <= 1 and (d == 0).mean() > 0.99
    else:
        hv = h.cpu().numpy()
        err = np.abs(hv.astype(np.float64) - h_ref.astype(np.float64))
        assert (err <= 8 * np.spacing(np.abs(h_ref)) + 1e-45).all()
    q_ref, s_ref, r_ref = oracle.quant_act(hv)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
    assert np.array_equal(r.cpu().numpy(), r_ref)


def test_ffn_gate_up_glu_down_matches_the_oracle():
    """x -> gate, up (one launch, shared quantisation) -> squared-ReLU GLU + quantisation -> down."""
    M, D, F = 4, 1024, 2816
    x, xf = activations(M, D, seed=31, dtype="bf16")
    Wg, Wu, Wd = weights(F, D, seed=32), weights(F, D, seed=33), weights(D, F, seed=34)
    (pg, gg, Tg), (pu, gu, Tu), (pd, gd, Td) = (oracle.pack_weights(W) for W in (Wg, Wu, Wd))
    yg = torch.empty((M, F), dtype=torch.bfloat16, device="cuda")
    yu = torch.empty((M, F), dtype=torch.bfloat16, device="cuda")
    layers = [tb.Layer(dev(pg), dev(np.array([gg], np.float32)), x, yg),
              tb.Layer(dev(pu), dev(np.array([gu], np.float32)), x, yu)]
    tb.layer_chain(layers)
    xq, s, r = tb.glu_quant(yg, yu, tb.GLU_RELU2)
    y, acc = tb.forward_quantized(dev(pd), dev(np.array([gd], np.float32)), xq, s, r, out_dtype=torch.bfloat16,
                                  acc_out=True)
    # oracle: the two products, stored as bf16, the gated activation, its codes, the down product
    _, yg_ref, *_ = oracle.forward(Tg, gg, xf)
    _, yu_ref, *_ = oracle.forward(Tu, gu, xf)
    to_bf16 = lambda v: (oracle.round_bf16(v).astype(np.uint32) << 16).view(np.float32)
    h_ref, q_ref, s_ref, r_ref = oracle.glu_quant(to_bf16(yg_ref), to_bf16(yu_ref), oracle.GLU_RELU2, True)
    acc_ref = oracle.accumulate(q_ref, Td)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_y_matches(y, oracle.dequant(acc_ref, gd, s_ref), acc_ref)


def test_glu_rejects_unknown_activation():
    g = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tb.BitLinearError) as e:
        tb.glu_quant(g, g, 7)
    assert e.value.code == tb.BL_ERR_INVALID_ARG


# ----------------------------------------------------------------------------
# The lookup-table decode product: the same exact accumulators as the
# forward (bit for bit), y at the forward's bars, and equal to the
# tensor-core decode kernel's output on the same codes.
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(6912, 2560), (2560, 2560), (1000, 8192), (300, 24576), (17, 64), (333, 8640)])
def test_lut_product_parity(N, K):
    W = weights(N, K, seed=N + K)
    packed_ref, gamma_ref, T = oracle.pack_weights(W)
    x, xf = activations(1, K, seed=K, dtype="bf16")
    acc_ref, y_ref, *_ = oracle.forward(T, gamma_ref, xf)
    p, g = dev(packed_ref), dev(np.array([gamma_ref], np.float32))
    xq, s, r = tb.quant_act(x)
    for ydt in (torch.bfloat16, torch.float32):
        y, acc = tb.forward_lut(p, g, xq, s, r, out_dtype=ydt, acc_out=True)
        assert np.array_equal(acc.cpu().numpy(), acc_ref)
        assert_y_matches(y, y_ref, acc_ref)
    if K % 128 == 0:
        y2 = tb.forward_quantized(p, g, xq, s, r, out_dtype=torch.bfloat16)
        y1 = tb.forward_lut(p, g, xq, s, r, out_dtype=torch.bfloat16)
        assert torch.equal(y1, y2)


def test_lut_product_extremes():
    """All weights +1 or -1 and a token at +-127: |acc| = 127 K through the tables."""
    N, K = 64, 4096
    for sign in (1, -1):
        T = np.full((N, K), sign, np.int8)
        packed = dev(oracle.pack(T))
        xq = torch.full((1, K), 127, dtype=torch.int8, device="cuda")
        s = torch.ones(1, dtype=torch.float32, device="cuda")
        r = torch.full((1,), 127 * K, dtype=torch.int32, device="cuda")
        g = torch.ones(1, dtype=torch.float32, device="cuda")
        y, acc = tb.forward_lut(packed, g, xq, s, r, out_dtype=torch.float32, acc_out=True)
        assert (acc.cpu().numpy() == sign * 127 * K).all()


def test_lut_product_rejects_unsupported_shapes():
    p = torch.zeros((8, 64), dtype=torch.uint8, device="cuda")
    g = torch.ones(1, dtype=torch.float32, device="cuda")
    for M, K in ((2, 256), (1, 24576 + 64)):
        xq = torch.zeros((M, K), dtype=torch.int8, device="cuda")
        pk = torch.zeros((8, K // 4), dtype=torch.uint8, device="cuda")
        s = torch.ones(M, dtype=torch.float32, device="cuda")
        r = torch.zeros(M, dtype=torch.int32, device="cuda")
        with pytest.raises(tb.BitLinearError) as e:
            tb.forward_lut(pk, g, xq, s, r)
        assert e.value.code == tb.BL_ERR_UNSUPPORTED_SHAPE


# ----------------------------------------------------------------------------
# The straight-through backward.  The operands are exact on both sides (bf16
# dy as given, t in {-1, 0, 1}, xhat = bf16(q / s) formed the same way), the
# products of bf16 pairs are exact in fp32, so the only error is the fp32
# accumulation over the R summed terms: |err| <= R * 2^-24 * sum|terms| for
# any order of the sums (each partial sum rounded once).
# ----------------------------------------------------------------------------

def _ste_inputs(M, N, K, seed):
    W = weights(N, K, seed=seed)
    packed_ref, gamma_ref, T = oracle.pack_weights(W)
    x, xf = activations(M, K, seed=seed + 1, dtype="bf16")
    dy_bits, dyf = synth.activations_bf16(M, N, seed=seed + 2)
    return packed_ref, gamma_ref, T, x, xf, bf16_dev(dy_bits), dyf


def _assert_within_accumulation_bound(got, ref, absterms, R):
    bound = max(R * 2.0 ** -24, 1e-6) * absterms + 1e-30
    err = np.abs(got.astype(np.float64) - ref)
    assert (err <= bound).all(), "max err/bound %.3g" % float((err / bound).max())


@pytest.mark.parametrize("M,N,K", [(8, 64, 64), (64, 640, 1024), (256, 512, 2560), (136, 320, 192)])
def test_ste_backward_parity(M, N, K):
    packed_ref, gamma_ref, T, x, xf, dy, dyf = _ste_inputs(M, N, K, seed=M + N + K)
    p, g = dev(packed_ref), dev(np.array([gamma_ref], np.float32))
    xq, s, _ = tb.quant_act(x)
    dx, dw = tb.ste_backward(p, g, K, dy, xq, s)
    q_ref, s_ref, _ = oracle.quant_act(xf)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    dx_ref = oracle.ste_grad_input(dyf, T, gamma_ref)
    absx = float(gamma_ref) * (np.abs(dyf).astype(np.float64) @ np.abs(T).astype(np.float64))
    _assert_within_accumulation_bound(dx.cpu().numpy(), dx_ref, absx, N)
    xhat = oracle.ste_xhat(q_ref, s_ref)
    dw_ref = oracle.ste_grad_weight(dyf, xhat)
    absw = np.abs(dyf).astype(np.float64).T @ np.abs(xhat).astype(np.float64)
    _assert_within_accumulation_bound(dw.cpu().numpy(), dw_ref, absw, M)


def test_ste_backward_bf16_dx_and_skips():
    M, N, K = 64, 256, 512
    packed_ref, gamma_ref, T, x, xf, dy, dyf = _ste_inputs(M, N, K, seed=5)
    p, g = dev(packed_ref), dev(np.array([gamma_ref], np.float32))
    xq, s, _ = tb.quant_act(x)
    dx32, _ = tb.ste_backward(p, g, K, dy, xq, s, dw=False)
    dx16, none = tb.ste_backward(p, g, K, dy, xq, s, dx_dtype=torch.bfloat16, dw=False)
    assert none is None
    # bf16 dx is the kernel's fp32 dx rounded once
    want = (f32_bits(dx32.cpu().numpy()) >> 16) + ((f32_bits(dx32.cpu().numpy()) >> 15) & 1)
    d = np.abs(bf16_bits(dx16).astype(np.int64) - want.astype(np.int64))
    assert d.max() <= 1
    _, dw_only = tb.ste_backward(p, g, K, dy, xq, s, dx=False)
    assert dw_only is not None and dw_only.shape == (N, K)


def test_ste_gradient_matches_the_forward():
    """<dx, xhat> = <dy, y_acc * gamma / s>: the backward of the forward's own bilinear form."""
    M, N, K = 64, 768, 2560
    packed_ref, gamma_ref, T, x, xf, dy, dyf = _ste_inputs(M, N, K, seed=9)
    p, g = dev(packed_ref), dev(np.array([gamma_ref], np.float32))
    xq, s, r = tb.quant_act(x)
    y = tb.forward_quantized(p, g, xq, s, r, out_dtype=torch.float32)
    dx, _ = tb.ste_backward(p, g, K, dy, xq, s, dw=False)
    q_ref, s_ref, _ = oracle.quant_act(xf)
    xhat = (q_ref.astype(np.float64) / s_ref[:, None].astype(np.float64))
    lhs = float(np.sum(dx.cpu().numpy().astype(np.float64) * xhat))
    rhs = float(np.sum(dyf.astype(np.float64) * y.cpu().numpy().astype(np.float64)))
    assert abs(lhs - rhs) <= 1e-4 * float(np.sum(np.abs(dyf.astype(np.float64) * y.cpu().numpy().astype(np.float64))))


def test_ste_rejects_unsupported_shapes():
    p = torch.zeros((96, 16), dtype=torch.uint8, device="cuda")
    g = torch.ones(1, dtype=torch.float32, device="cuda")
    dy = torch.zeros((8, 96), dtype=torch.bfloat16, device="cuda")
    xq = torch.zeros((8, 64), dtype=torch.int8, device="cuda")
    s = torch.ones(8, dtype=torch.float32, device="cuda")
    with pytest.raises(tb.BitLinearError) as e:
        tb.ste_backward(p, g, 64, dy, xq, s)  # N = 96 is not a multiple of 64
    assert e.value.code == tb.BL_ERR_UNSUPPORTED_SHAPE
