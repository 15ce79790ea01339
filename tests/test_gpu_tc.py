"""The tensor-core form of the decode product (2 to 16 tokens on int8 codes:
tcgen05.mma kind::i8 with the unpacked ternary codes in tensor memory)
against the oracle, and against the CUDA-core form bit for bit.

"BitNet's Real Bet: Designing the Whole Inference Stack", section "A low-bit
model is a whole-stack design" (packed weights unpacked on chip, computed
with 8-bit activations); the sums are exact int32, so the accumulators are
compared bit for bit and the outputs at the output bar.
"""
import numpy as np
import pytest
import torch

import oracle
import ternary_weight_a8_b200 as tb
from parity import activations, assert_y_matches, dev, weights

pytestmark = pytest.mark.gpu


@pytest.fixture
def form():
    """The decode form forced on this thread, reset afterwards."""
    yield tb.set_decode_form
    tb.set_decode_form(tb.DECODE_FORM_AUTO)


# One layer: N from under one 128-row unit to ragged unit counts, K from one
# 128-input block to several 512-input stages with a partial last stage.
SINGLE = [(9, 129, 128), (12, 300, 1024), (16, 1000, 1152), (13, 640, 2560), (16, 2048, 4096), (10, 77, 8704),
          (2, 500, 1024), (8, 384, 2176)]


@pytest.mark.parametrize("M,N,K", SINGLE)
@pytest.mark.parametrize("ydtype", [torch.bfloat16, torch.float32])
def test_tensor_core_decode_matches_the_oracle(M, N, K, ydtype, form):
    form(tb.DECODE_FORM_TENSOR_CORES)
    x, xf = activations(M, K, seed=M * 7 + K, dtype="bf16")
    xq, sc, rs = tb.quant_act(x)
    packed, gamma, T = oracle.pack_weights(weights(N, K, seed=N + K))
    y, acc = tb.forward_quantized(dev(packed), dev(np.array([gamma], np.float32)), xq, sc, rs, out_dtype=ydtype,
                                  acc_out=True)
    acc_ref, y_ref, *_ = oracle.forward(T, gamma, xf)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_y_matches(y, y_ref, acc_ref)


def test_tensor_core_group_of_layers_matches_the_oracle(form):
    """Several layers of different K and their own codes in one launch (longest K
    first), more units than SMs so that units are handed out by ticket."""
    form(tb.DECODE_FORM_TENSOR_CORES)
    M = 16
    specs = [(640, 9000), (2048, 12000), (1152, 333), (4096, 7000)]
    layers, refs = [], []
    for i, (K, N) in enumerate(specs):
        x, xf = activations(M, K, seed=40 + i, dtype="bf16")
        xq, sc, rs = tb.quant_act(x)
        packed, gamma, T = oracle.pack_weights(weights(N, K, seed=50 + i))
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
        layers.append(tb.Layer(dev(packed), dev(np.array([gamma], np.float32)), None, y, xq=xq, scale=sc,
                               rowsum=rs, acc_out=acc))
        refs.append(oracle.forward(T, gamma, xf))
    for _ in range(2):  # twice: the ticket counter is reset by each launch
        tb.layer_chain(layers)
        for L, (acc_ref, y_ref, *_) in zip(layers, refs):
            assert np.array_equal(L.acc_out.cpu().numpy(), acc_ref)
            assert_y_matches(L.y, y_ref, acc_ref)


@pytest.mark.parametrize("M", [3, 8, 9, 16])
def test_tensor_core_equals_cuda_core_form(M, form):
    """The same group through both forms: identical outputs and accumulators."""
    K = 8192
    specs = [(K, 4096), (K, 4096), (28672, 1024)]
    xs = [activations(M, k, seed=60 + i, dtype="bf16")[0] for i, (k, _) in enumerate(specs)]
    ws = [tb.pack_weights(dev(weights(n, k, seed=70 + i))) for i, (k, n) in enumerate(specs)]
    out = {}
    for f in (tb.DECODE_FORM_CUDA_CORES, tb.DECODE_FORM_TENSOR_CORES):
        form(f)
        layers = []
        for (k, n), x, (p, g) in zip(specs, xs, ws):
            layers.append(tb.Layer(p, g, x, torch.empty((M, n), dtype=torch.bfloat16, device="cuda"),
                                   acc_out=torch.empty((M, n), dtype=torch.int32, device="cuda")))
        tb.layer_chain(layers)
        out[f] = [(L.y, L.acc_out) for L in layers]
    for (y1, a1), (y2, a2) in zip(out[tb.DECODE_FORM_CUDA_CORES], out[tb.DECODE_FORM_TENSOR_CORES]):
        assert torch.equal(a1, a2)
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_tensor_core_extremes(form):
    """|acc| at its largest: all weights +1 or -1 against codes of +-127."""
    form(tb.DECODE_FORM_TENSOR_CORES)
    M, N, K = 16, 256, 4096
    W = np.where(np.arange(N)[:, None] % 2 == 0, 1.0, -1.0).astype(np.float32) * np.ones((N, K), np.float32)
    x = np.where(np.arange(M)[:, None] % 3 == 0, 1.0, -1.0).astype(np.float32) * np.ones((M, K), np.float32)
    packed, gamma, T = oracle.pack_weights(W)
    xq, sc, rs = tb.quant_act(dev(x))
    y, acc = tb.forward_quantized(dev(packed), dev(np.array([gamma], np.float32)), xq, sc, rs,
                                  out_dtype=torch.float32, acc_out=True)
    acc_ref, y_ref, *_ = oracle.forward(T, gamma, x)
    assert np.abs(acc_ref).max() == 127 * K
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert_y_matches(y, y_ref, acc_ref)

