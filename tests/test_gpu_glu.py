"""The FFN's gate and up BitLinears fused with the gated activation and the
quantisation of its result (bitlinear_gate_up_glu), against the oracle.

"BitNet's Real Bet: Designing the Whole Inference Stack", native-training
section (SwiGLU for the 2024 model, squared ReLU for 2B4T); "A Two-Billion
Ternary Bet" (squared-ReLU-style activations).  The gate and up outputs are
floating point (within the output bar of the oracle's exact values), and h
and its codes are decided from them, so the oracle takes those decisions on
the same values: the gate and up outputs as the library stores them
(``layer_chain``, itself checked against ``oracle.forward`` at the bar, and
bit-identical to what the fused path forms internally), then
``oracle.glu_quant``, then the down product on the codes.  Squared ReLU is
exact fp32 arithmetic, so h, the codes, scales, code sums and the down
product's int32 accumulators are compared bit for bit; SiLU calls the device
``expf``, so h is held to one bf16 ulp (8 fp32 ulps) and the codes are
compared with the oracle's quantisation of the kernel's own h.  Decode sizes
run as one launch that forms and quantises h itself; larger M through the
tensor-core path.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_a8_b200 as tb
from parity import activations, assert_y_matches, bf16_bits, dev, f32_bits, weights

pytestmark = pytest.mark.gpu


def _values(t):
    """A device tensor of bf16 or fp32 values as fp32 numpy values."""
    if t.dtype == torch.bfloat16:
        return (bf16_bits(t).astype(np.uint32) << 16).view(np.float32)
    return t.cpu().numpy()


def _ffn(M, N, K, dtype, seed):
    """Weights and input of a gate/up pair; the stored gate and up outputs (the
    library's, checked against the oracle at the output bar) as fp32 values."""
    x, xf = activations(M, K, seed=seed, dtype=dtype)
    Wg, Wu = weights(N, K, seed=seed + 1), weights(N, K, seed=seed + 2)
    (pg, gg, Tg), (pu, gu, Tu) = oracle.pack_weights(Wg), oracle.pack_weights(Wu)
    dev_w = (dev(pg), dev(np.array([gg], np.float32)), dev(pu), dev(np.array([gu], np.float32)))
    ydt = torch.bfloat16 if dtype == "bf16" else torch.float32
    yg = torch.empty((M, N), dtype=ydt, device="cuda")
    yu = torch.empty((M, N), dtype=ydt, device="cuda")
    tb.layer_chain([tb.Layer(dev_w[0], dev_w[1], x, yg), tb.Layer(dev_w[2], dev_w[3], x, yu)])
    for y, T, g in ((yg, Tg, gg), (yu, Tu, gu)):
        acc_ref, y_ref, *_ = oracle.forward(T, g, xf)
        assert_y_matches(y, y_ref, acc_ref)
    return x, dev_w, _values(yg), _values(yu)


# Decode sizes: 1 to 8 tokens in one launch (N past one unit, ragged unit
# counts, and 8 x 114688, whose 512-element quantisation slices outnumber
# the grid's warps; at one token 16-row units over 2048-input stages: four
# units, K not a multiple of 2048, and more units than resident blocks), 9 to 16
# tokens as the products then the gated-activation kernel; and many tokens
# (the tensor-core GEMM whose
# tiles pair gate and up rows: one CTA up to 128 tokens, CTA pairs beyond,
# ragged M, N (not a multiple of the 128-column tile) and K).
RELU2 = [(1, 1024, 1024, "bf16"), (1, 2816, 2560, "bf16"), (3, 704, 4096, "f32"), (8, 2816, 1024, "bf16"),
         (16, 1088, 2048, "bf16"), (1, 6912, 2560, "bf16"), (40, 704, 512, "bf16"), (2048, 1024, 512, "bf16"),
         (300, 1088, 576, "f32"), (513, 704, 320, "bf16"), (8, 114688, 128, "bf16"), (9, 1088, 1024, "f32"),
         (12, 2816, 2560, "bf16"), (1, 1088, 3072, "bf16"), (1, 64, 8192, "bf16"), (1, 4160, 640, "f32"),
         (1, 28736, 1024, "bf16")]


@pytest.mark.parametrize("M,N,K,dtype", RELU2)
def test_gate_up_glu_relu2_matches_the_oracle(M, N, K, dtype):
    x, (pg, gg, pu, gu), yg, yu = _ffn(M, N, K, dtype, seed=M + N + K)
    h, xq, s, r = tb.gate_up_glu(pg, gg, pu, gu, x, tb.GLU_RELU2, h=True)
    h_ref, q_ref, s_ref, r_ref = oracle.glu_quant(yg, yu, oracle.GLU_RELU2, dtype == "bf16")
    assert np.array_equal(f32_bits(_values(h)), f32_bits(h_ref))
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
    assert np.array_equal(r.cpu().numpy(), r_ref)


@pytest.mark.parametrize("M,N,K,dtype", [(1, 2816, 2560, "bf16"), (5, 1024, 1024, "f32"), (16, 704, 4096, "bf16"),
                                         (64, 512, 512, "bf16")])
def test_gate_up_glu_silu_at_its_bar(M, N, K, dtype):
    x, (pg, gg, pu, gu), yg, yu = _ffn(M, N, K, dtype, seed=7 * M + N)
    h, xq, s, r = tb.gate_up_glu(pg, gg, pu, gu, x, tb.GLU_SILU, h=True)
    h_ref = oracle.glu(yg, yu, oracle.GLU_SILU, dtype == "bf16")
    got = _values(h)
    if dtype == "bf16":
        from parity import bf16_ordered
        d = np.abs(bf16_ordered(bf16_bits(h)).astype(np.int64) -
                   bf16_ordered((f32_bits(h_ref) >> 16).astype(np.uint16)).astype(np.int64))
        assert d.max() <= 1
    else:
        d = np.abs(f32_bits(got).astype(np.int64) - f32_bits(h_ref).astype(np.int64))
        assert d.max() <= 8
    q_ref, s_ref, r_ref = oracle.quant_act(got)  # the integer decision on the kernel's own h
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
    assert np.array_equal(r.cpu().numpy(), r_ref)


@pytest.mark.parametrize("M", [1, 8, 2048])
def test_ffn_through_the_fused_path_matches_the_oracle(M):
    """x -> gate, up, squared-ReLU h and its codes (one call) -> down: the down
    product's int32 accumulators bit for bit, its output at the bf16 bar."""
    D, F = (1024, 2816) if M < 2048 else (512, 1024)
    x, (pg, gg, pu, gu), yg, yu = _ffn(M, F, D, "bf16", seed=100 + M)
    Wd = weights(D, F, seed=200 + M)
    pd, gd, Td = oracle.pack_weights(Wd)
    xq, s, r = tb.gate_up_glu(pg, gg, pu, gu, x, tb.GLU_RELU2)
    y, acc = tb.forward_quantized(dev(pd), dev(np.array([gd], np.float32)), xq, s, r, acc_out=True)
    _, q_ref, s_ref, _ = oracle.glu_quant(yg, yu, oracle.GLU_RELU2, True)
    acc_ref = oracle.accumulate(q_ref, Td)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_y_matches(y, oracle.dequant(acc_ref, gd, s_ref), acc_ref)


@pytest.mark.parametrize("M", [1, 8, 16])
@pytest.mark.parametrize("act", [tb.GLU_RELU2, tb.GLU_SILU])
def test_fused_equals_chain_then_glu_quant(M, act):
    """The one-launch path and the separate launches give identical bits (the
    70B-class FFN width)."""
    N, K = 28672, 8192
    x, _ = activations(M, K, seed=M, dtype="bf16")
    pg, gg = tb.pack_weights(dev(weights(N, K, seed=41)))
    pu, gu = tb.pack_weights(dev(weights(N, K, seed=42)))
    yg = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    yu = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    tb.layer_chain([tb.Layer(pg, gg, x, yg), tb.Layer(pu, gu, x, yu)])
    h1, q1, s1, r1 = tb.glu_quant(yg, yu, act, h=True)
    for _ in range(2):  # a second call on the same (cached) workspace
        h2, q2, s2, r2 = tb.gate_up_glu(pg, gg, pu, gu, x, act, h=True)
        assert torch.equal(h1.view(torch.int16), h2.view(torch.int16))
        assert torch.equal(q1, q2) and torch.equal(s1, s2) and torch.equal(r1, r2)


def test_gate_up_glu_ignores_a_forced_split():
    """The fused call spreads its quantisation over the warps of its grid and
    never splits along K; a forced split on the calling thread leaves its
    result unchanged."""
    M, N, K = 4, 1088, 5120
    x, (pg, gg, pu, gu), yg, yu = _ffn(M, N, K, "bf16", seed=55)
    want = tb.gate_up_glu(pg, gg, pu, gu, x, tb.GLU_RELU2)
    tb.set_decode_split(4)
    try:
        got = tb.gate_up_glu(pg, gg, pu, gu, x, tb.GLU_RELU2)
    finally:
        tb.set_decode_split(0)
    for a, b in zip(want, got):
        assert torch.equal(a, b)
    _, q_ref, s_ref, r_ref = oracle.glu_quant(yg, yu, oracle.GLU_RELU2, True)
    assert np.array_equal(got[0].cpu().numpy(), q_ref)
    assert np.array_equal(f32_bits(got[1].cpu().numpy()), f32_bits(s_ref))
    assert np.array_equal(got[2].cpu().numpy(), r_ref)


def test_gate_up_glu_zero_input_and_status():
    M, N, K = 2, 640, 1024
    pg, gg = tb.pack_weights(dev(weights(N, K, seed=1)))
    pu, gu = tb.pack_weights(dev(weights(N, K, seed=2)))
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    ws = tb.new_workspace(tb.gate_up_glu_workspace_bytes(M, N, K))
    h, xq, s, r = tb.gate_up_glu(pg, gg, pu, gu, x, tb.GLU_RELU2, h=True, workspace=ws)
    assert (h.float() == 0).all() and (xq == 0).all() and (r == 0).all()
    _, s_ref, _ = oracle.quant_act(np.zeros((M, N), np.float32))  # the 1e-5 floor
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
    assert tb.device_status(ws) == tb.BL_OK


def test_gate_up_glu_rejects_bad_arguments():
    pg = torch.zeros((96, 16), dtype=torch.uint8, device="cuda")
    g = torch.ones(1, dtype=torch.float32, device="cuda")
    x = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tb.BitLinearError) as e:  # N = 96: not a multiple of 64
        tb.gate_up_glu(pg, g, pg, g, x)
    assert e.value.code == tb.BL_ERR_UNSUPPORTED_SHAPE
    pg = torch.zeros((128, 16), dtype=torch.uint8, device="cuda")
    with pytest.raises(tb.BitLinearError) as e:
        tb.gate_up_glu(pg, g, pg, g, x, act=5)
    assert e.value.code == tb.BL_ERR_INVALID_ARG
