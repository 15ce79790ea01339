"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Every case draws seeded synthetic inputs once, hands the same arrays to both
sides, and compares at the bars stated in ``parity.py``: packed weights,
gamma, int8 activations, scales, row sums and int32 accumulators bit for bit;
outputs within 1e-6 relative (fp32) or 1 ulp (bf16).  Sizes span several
tiles with ragged tails; the full-size workloads of the pages (2B/3B decode,
2B prefill, 70B layer chain) are checked on sampled output rows, which the
oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import ternary_weight_a8_b200 as tb
from conftest import read_golden
from parity import activations, assert_y_matches, bf16_dev, dev, f32_bits, weights

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _auto_path():
    tb.set_path(tb.PATH_AUTO)
    yield
    tb.set_path(tb.PATH_AUTO)


# ----------------------------------------------------------------------------
# offline weight path: gamma + ternarise + pack
# ----------------------------------------------------------------------------

PACK_SHAPES = [(1, 64), (17, 192), (33, 640), (256, 256), (6912, 2560), (2560, 2560), (8640, 3200),
               (3200, 8640), (10240, 8192), (28672, 8192), (8192, 28672)]


@pytest.mark.parametrize("N,K", PACK_SHAPES)
def test_pack_parity(N, K):
    W = weights(N, K, seed=N + K)
    packed_ref, gamma_ref, _ = oracle.pack_weights(W)
    packed, gamma = tb.pack_weights(dev(W))
    assert f32_bits(gamma.cpu().numpy())[0] == f32_bits([gamma_ref])[0]
    got = packed.cpu().numpy()
    if not np.array_equal(got, packed_ref):
        bad = np.argwhere(got != packed_ref)
        raise AssertionError("%d packed bytes differ, first at %s" % (len(bad), bad[:5].tolist()))


def _tie_matrix():
    """W whose mean magnitude makes some weights exactly (gamma + 1e-5) / 2 (and 3/2 of it)."""
    rng = np.random.default_rng(0)
    N, K = 64, 64
    signs = rng.choice([-1.0, 1.0], size=(N, K)).astype(np.float32)
    kind = rng.integers(0, 4, size=(N, K))  # 0: tie h, 1: c, 2: 3h, 3: c/3
    h = np.float32(0.2)
    for _ in range(60):
        mags = np.where(kind == 0, h, np.where(kind == 1, np.float32(0.5),
                        np.where(kind == 2, np.float32(3) * h, np.float32(0.5) / np.float32(3))))
        W = (signs * mags).astype(np.float32)
        g, _ = oracle.absmean_gamma(W)
        d = np.float32(g + np.float32(1e-5))
        h_new = np.float32(d * np.float32(0.5))
        if h_new == h:
            break
        h = h_new
    return W, h, d


def test_pack_exact_ties():
    W, h, d = _tie_matrix()
    assert float(h) * 2 == float(d)  # exact ties w / d = 0.5 by construction
    packed_ref, gamma_ref, T_ref = oracle.pack_weights(W)
    tie = np.abs(W) == h
    assert tie.sum() > 500 and (T_ref[tie] == 0).all()  # half rounds to the even neighbour 0
    packed, gamma = tb.pack_weights(dev(W))
    assert f32_bits(gamma.cpu().numpy())[0] == f32_bits([gamma_ref])[0]
    assert np.array_equal(packed.cpu().numpy(), packed_ref)


def test_pack_special_matrices():
    Z = np.zeros((8, 128), np.float32)
    packed, gamma = tb.pack_weights(dev(Z))
    assert gamma.item() == 0.0 and (packed.cpu().numpy() == 0x55).all()
    C = np.full((8, 128), -0.03, np.float32)
    packed, gamma = tb.pack_weights(dev(C))
    assert (packed.cpu().numpy() == 0x00).all()
    assert np.array_equal(packed.cpu().numpy(), oracle.pack_weights(C)[0])


# ----------------------------------------------------------------------------
# per-token activation quantisation
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("M,K,dtype", [(4, 256, "f32"), (3, 64, "f32"), (1, 2560, "bf16"), (16, 3200, "bf16"),
                                       (2048, 2560, "bf16"), (8, 28672, "bf16"), (5, 8640, "f32"),
                                       # many tokens, short and long rows
                                       (700, 2048, "f32"), (600, 576, "bf16"), (640, 4096, "bf16"),
                                       (600, 4160, "bf16"), (1200, 64, "f32"),
                                       # long tokens: one block up to 32768 inputs (a token in
                                       # registers), a cluster of CTAs per token beyond
                                       (1, 20480, "f32"), (2, 65536, "bf16"), (16, 16448, "bf16"),
                                       (1, 32768, "bf16"), (3, 40960, "bf16"), (1, 131072, "f32")])
def test_quant_parity(M, K, dtype):
    x, xf = activations(M, K, seed=M * 7 + K, dtype=dtype)
    q_ref, s_ref, r_ref = oracle.quant_act(xf)
    q, s, r = tb.quant_act(x)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
    assert np.array_equal(r.cpu().numpy(), r_ref)


def test_quant_golden_ties_and_degenerate_tokens():
    rows = read_golden("act_quant.txt")
    toks = [[float(v) for v in rows[i][1]] for i in range(0, len(rows), 4)]
    K = 64
    x = np.zeros((len(toks) + 2, K), np.float32)
    for i, t in enumerate(toks):
        x[i, :len(t)] = t
    x[-1, 5] = 3e-6  # below the 1e-5 floor
    q, s, r = tb.quant_act(dev(x))
    q_ref, s_ref, r_ref = oracle.quant_act(x)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(f32_bits(s.cpu().numpy()), f32_bits(s_ref))
    assert np.array_equal(r.cpu().numpy(), r_ref)
    for i in range(0, len(rows), 4):
        want = [int(v) for v in rows[i + 1][1]]
        assert q.cpu().numpy()[i // 4, :len(want)].tolist() == want


# ----------------------------------------------------------------------------
# the forward: acc bit-exact, y within the bar
# ----------------------------------------------------------------------------

def _full_case(M, N, K, xdtype, ydtype, path, seed=0):
    W = weights(N, K, seed=seed + 1)
    packed_ref, gamma_ref, T = oracle.pack_weights(W)
    x, xf = activations(M, K, seed=seed + 2, dtype=xdtype)
    acc_ref, y_ref, *_ = oracle.forward(T, gamma_ref, xf)
    tb.set_path(path)
    y, acc = tb.forward(dev(packed_ref), dev(np.array([gamma_ref], np.float32)), x,
                        out_dtype=ydtype, acc_out=True)
    got = acc.cpu().numpy()
    assert np.array_equal(got, acc_ref), "acc differs at %s" % np.argwhere(got != acc_ref)[:5].tolist()
    assert_y_matches(y, y_ref, acc_ref)


SMALL = [(1, 16, 64), (4, 256, 256), (3, 100, 192), (8, 300, 640), (9, 17, 128), (16, 1000, 320),
         (17, 300, 192), (100, 513, 384), (130, 260, 256), (256, 512, 1024)]


@pytest.mark.parametrize("M,N,K", [s for s in SMALL if s[0] <= 16])
@pytest.mark.parametrize("ydtype", [torch.float32, torch.bfloat16])
def test_forward_small_gemv(M, N, K, ydtype):
    _full_case(M, N, K, "bf16", ydtype, tb.PATH_GEMV, seed=M * N + K)


# One token takes the dp4a path of the decode kernel: K from one 64-input chunk
# to several 1024-input stages with a ragged last stage, N from one row to
# ragged 64-row units; fp32 inputs of K <= 2048 and bf16 inputs of K <= 9856
# (the most that fits beside a four-stage ring) are quantised inside the
# kernel, longer ones by the quantisation kernel.
ONE_TOKEN = [(1, 64), (63, 960), (65, 1024), (200, 1088), (130, 2048), (129, 4160), (64, 5120), (7, 8192),
             (300, 9856), (70, 9920)]


@pytest.mark.parametrize("N,K", ONE_TOKEN)
@pytest.mark.parametrize("xdtype", ["bf16", "f32"])
def test_forward_one_token(N, K, xdtype):
    _full_case(1, N, K, xdtype, torch.float32 if xdtype == "f32" else torch.bfloat16, tb.PATH_GEMV, seed=N + 7 * K)


# Layers with fewer 64-row units than SMs are split along K over the CTAs of a
# cluster (2 to 8, each a contiguous range of 1024-input stages) whose partial
# sums meet in one CTA's shared memory: one to 16 tokens, ragged N and K.
# Short, wide layers the decode kernel splits along K by itself; the last two
# take 5 and 3 CTAs per unit at one token (about 1.35 CTAs per SM).
KSPLIT = [(130, 3072), (64, 8192), (300, 2112), (17, 4160), (2560, 6912), (4096, 11008)]


@pytest.mark.parametrize("N,K", KSPLIT)
@pytest.mark.parametrize("M", [1, 2, 5, 9, 16])
def test_forward_ksplit(M, N, K):
    _full_case(M, N, K, "bf16", torch.bfloat16, tb.PATH_GEMV, seed=M + N + K)


@pytest.fixture
def forced_split():
    """The K-split forced to `ctas` CTAs per unit, reset afterwards."""
    def force(ctas):
        tb.set_decode_split(ctas)
    yield force
    tb.set_decode_split(0)


# The K-split forced on shapes the automatic choice leaves whole: both decode
# paths (dp4a for one token, mma.sync for more), activations quantised inside
# the kernel or streamed as codes, fp32 and bf16, up to the 8-CTA cluster.
FORCED = [(1, 640, 2048, "f32"), (1, 1000, 9216, "bf16"), (3, 2000, 4160, "bf16"), (8, 3000, 5120, "bf16"),
          (16, 1200, 8192, "f32"), (12, 1300, 2560, "bf16")]


@pytest.mark.parametrize("M,N,K,xdt", FORCED)
@pytest.mark.parametrize("ctas", [2, 3, 8])
def test_forward_forced_split(M, N, K, xdt, ctas, forced_split):
    forced_split(ctas)
    _full_case(M, N, K, xdt, torch.float32 if xdt == "f32" else torch.bfloat16, tb.PATH_GEMV, seed=M * K + ctas)


def test_forced_split_matches_unsplit_bit_for_bit(forced_split):
    """The split changes the order of integer sums only: acc and y are identical."""
    W = weights(700, 8192, seed=11)
    packed, gamma = tb.pack_weights(dev(W))
    for M in (1, 4, 16):
        x, _ = activations(M, 8192, seed=M + 3, dtype="bf16")
        forced_split(1)
        y1, a1 = tb.forward(packed, gamma, x, acc_out=True, out_dtype=torch.float32)
        for ctas in (2, 5, 8):
            forced_split(ctas)
            y2, a2 = tb.forward(packed, gamma, x, acc_out=True, out_dtype=torch.float32)
            assert torch.equal(a1, a2) and torch.equal(y1, y2)


@pytest.mark.parametrize("M,N,K", SMALL)
@pytest.mark.parametrize("ydtype", [torch.float32, torch.bfloat16])
def test_forward_small_gemm(M, N, K, ydtype):
    _full_case(M, N, K, "f32", ydtype, tb.PATH_GEMM, seed=M + N + K)


def test_forward_single_256_both_paths():
    """K = N = 256, 4 tokens, fp32 in and out (seed 0)."""
    for path in (tb.PATH_GEMV, tb.PATH_GEMM, tb.PATH_AUTO):
        _full_case(4, 256, 256, "f32", torch.float32, path, seed=0)


@pytest.mark.parametrize("N", [6912, 2560])
def test_forward_decode_2b(N):
    _full_case(1, N, 2560, "bf16", torch.bfloat16, tb.PATH_AUTO, seed=N)


@pytest.mark.parametrize("K,N", [(3200, 8640), (8640, 3200)])
@pytest.mark.parametrize("M", [1, 2, 4, 8, 16])
def test_forward_decode_3b_sweep(K, N, M):
    _full_case(M, N, K, "bf16", torch.bfloat16, tb.PATH_AUTO, seed=K + M)


def _sampled_case(M, N, K, rows, seed, xdtype="bf16", ydtype=torch.bfloat16, path=tb.PATH_AUTO):
    """Full-size run on the GPU; the oracle computes the sampled output rows only."""
    W = weights(N, K, seed=seed)
    gamma_ref, _ = oracle.absmean_gamma(W)
    Wd = dev(W)
    packed, gamma = tb.pack_weights(Wd)
    del Wd
    assert f32_bits(gamma.cpu().numpy())[0] == f32_bits([gamma_ref])[0]
    x, xf = activations(M, K, seed=seed + 1, dtype=xdtype)
    tb.set_path(path)
    y, acc = tb.forward(packed, gamma, x, out_dtype=ydtype, acc_out=True)
    T_rows = oracle.ternarize(W[rows], gamma_ref)
    acc_ref, y_ref, *_ = oracle.forward(T_rows, gamma_ref, xf)
    got = acc.cpu().numpy()[:, rows]
    assert np.array_equal(got, acc_ref)
    assert_y_matches(y[:, torch.as_tensor(rows, device=y.device)].contiguous(), y_ref, acc_ref)
    # whole-output properties: finite, and zero exactly where acc is zero
    yf = y.float()
    assert torch.isfinite(yf).all()
    assert ((acc == 0) == (yf == 0)).all()


def test_forward_prefill_2b_sampled():
    rng = np.random.default_rng(4)
    rows = np.sort(np.concatenate([rng.choice(6912, 120, replace=False), [0, 255, 256, 6911]]))
    _sampled_case(2048, 6912, 2560, np.unique(rows), seed=40)


def test_forward_prefill_ragged_full():
    """A prefill shape with ragged M, N and K tails, checked everywhere."""
    _full_case(300, 1000, 576, "bf16", torch.bfloat16, tb.PATH_AUTO, seed=77)


@pytest.mark.parametrize("M,N,K,ydtype", [(300, 1000, 576, torch.bfloat16), (300, 1000, 576, torch.float32),
                                          (513, 772, 320, torch.float32), (2048, 512, 256, torch.bfloat16),
                                          (700, 520, 192, torch.bfloat16)])
def test_forward_y_only_many_tokens(M, N, K, ydtype):
    """Without the accumulator output (the serving call), checked everywhere."""
    seed = M + N
    W = weights(N, K, seed=seed)
    packed_ref, gamma_ref, T = oracle.pack_weights(W)
    x, xf = activations(M, K, seed=seed + 1, dtype="bf16")
    acc_ref, y_ref, *_ = oracle.forward(T, gamma_ref, xf)
    tb.set_path(tb.PATH_AUTO)
    y = tb.forward(dev(packed_ref), dev(np.array([gamma_ref], np.float32)), x, out_dtype=ydtype)
    assert_y_matches(y, y_ref, acc_ref)


@pytest.mark.parametrize("K", [2560, 8640])
def test_forward_quantized_matches_forward(K):
    W = weights(640, K, seed=5)
    packed, gamma = tb.pack_weights(dev(W))
    for M in (1, 8, 16, 64):
        x, _ = activations(M, K, seed=M, dtype="bf16")
        y1, a1 = tb.forward(packed, gamma, x, acc_out=True)
        xq, s, r = tb.quant_act(x)
        y2, a2 = tb.forward_quantized(packed, gamma, xq, s, r, acc_out=True)
        assert torch.equal(a1, a2) and torch.equal(y1, y2)


def test_gemv_and_gemm_agree_on_decode_sizes():
    W = weights(3200, 8640, seed=9)
    packed, gamma = tb.pack_weights(dev(W))
    for M in (1, 5, 16):
        x, _ = activations(M, 8640, seed=M + 100, dtype="bf16")
        tb.set_path(tb.PATH_GEMV)
        y1, a1 = tb.forward(packed, gamma, x, acc_out=True, out_dtype=torch.float32)
        tb.set_path(tb.PATH_GEMM)
        y2, a2 = tb.forward(packed, gamma, x, acc_out=True, out_dtype=torch.float32)
        assert torch.equal(a1, a2) and torch.equal(y1, y2)


def test_forward_extreme_accumulators():
    """|acc| = 127 * K at K = 28672 (all weights +1, every activation code 127) stays exact."""
    K, N = 28672, 64
    W = np.full((N, K), 0.02, np.float32)
    W[1::2] *= -1
    packed, gamma = tb.pack_weights(dev(W))
    x = torch.full((3, K), 2.5, dtype=torch.bfloat16, device="cuda")
    for path in (tb.PATH_GEMV, tb.PATH_GEMM):
        tb.set_path(path)
        y, acc = tb.forward(packed, gamma, x, acc_out=True, out_dtype=torch.float32)
        a = acc.cpu().numpy()
        assert (a[:, 0::2] == 127 * K).all() and (a[:, 1::2] == -127 * K).all()
        want = 127 * K * float(np.float32(0.02)) / float(np.float32(127 / 2.5))
        assert np.allclose(y.cpu().numpy()[:, 0], want, rtol=1e-6)


def test_forward_zero_tokens_and_weights():
    W = weights(300, 512, seed=3)
    packed, gamma = tb.pack_weights(dev(W))
    x = torch.zeros((20, 512), dtype=torch.bfloat16, device="cuda")
    x[3, 7] = 1.0
    for path in (tb.PATH_GEMM,):
        tb.set_path(path)
        y, acc = tb.forward(packed, gamma, x, acc_out=True)
        assert (acc[torch.arange(20) != 3] == 0).all() and (y.float()[torch.arange(20) != 3] == 0).all()
    packed0, gamma0 = tb.pack_weights(torch.zeros((300, 512), device="cuda"))
    y, acc = tb.forward(packed0, gamma0, x[:4], acc_out=True)
    assert (acc == 0).all() and (y.float() == 0).all()


# ----------------------------------------------------------------------------
# 70B-class layer chain at decode
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("M", [1, 8, 16])
def test_layer_chain_70b_sampled(M):
    """The five BitLinears of a 70B-class block in one grouped launch (split into
    items of a few stages), with every layer's int32 accumulators compared bit
    for bit on sampled rows."""
    layers_shape = synth.CHAIN_70B
    shared = synth.CHAIN_70B_SHARED_INPUT
    rng = np.random.default_rng(M)
    layers, refs = [], []
    x_prev = None
    for li, (K, N) in enumerate(layers_shape):
        W = weights(N, K, seed=1000 + li)  # re-randomised per layer from a seed
        gamma_ref, _ = oracle.absmean_gamma(W)
        Wd = dev(W)
        packed, gamma = tb.pack_weights(Wd)
        del Wd
        assert f32_bits(gamma.cpu().numpy())[0] == f32_bits([gamma_ref])[0]
        if shared[li]:
            x, xf = x_prev
        else:
            x, xf = activations(M, K, seed=2000 + li, dtype="bf16")
        x_prev = (x, xf)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        acc = torch.full((M, N), -7, dtype=torch.int32, device="cuda")
        layers.append(tb.Layer(packed, gamma, x, y, acc_out=acc))
        rows = np.unique(np.concatenate([rng.choice(N, 48, replace=False), [0, 63, 64, N - 1]]))
        T_rows = oracle.ternarize(W[rows], gamma_ref)
        acc_ref, y_ref, *_ = oracle.forward(T_rows, gamma_ref, xf)
        refs.append((rows, acc_ref, y_ref))
        del W
    tb.layer_chain(layers)
    torch.cuda.synchronize()
    for L, (rows, acc_ref, y_ref) in zip(layers, refs):
        idx = torch.as_tensor(rows, device="cuda")
        assert np.array_equal(L.acc_out[:, idx].cpu().numpy(), acc_ref)
        assert_y_matches(L.y[:, idx].contiguous(), y_ref, acc_ref)
        assert torch.isfinite(L.y.float()).all()
        assert ((L.acc_out == 0) == (L.y.float() == 0)).all()


@pytest.mark.parametrize("M", [1, 16])
def test_layer_chain_3b_full(M):
    """Both 3B-class BitLinears as one chain call, every output and accumulator compared."""
    layers, refs = [], []
    for li, (K, N) in enumerate([(3200, 8640), (8640, 3200)]):
        W = weights(N, K, seed=3000 + li)
        packed_ref, gamma_ref, T = oracle.pack_weights(W)
        x, xf = activations(M, K, seed=3100 + li, dtype="bf16")
        acc_ref, y_ref, *_ = oracle.forward(T, gamma_ref, xf)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
        layers.append(tb.Layer(dev(packed_ref), dev(np.array([gamma_ref], np.float32)), x, y, acc_out=acc))
        refs.append((acc_ref, y_ref))
    tb.layer_chain(layers)
    for L, (acc_ref, y_ref) in zip(layers, refs):
        assert np.array_equal(L.acc_out.cpu().numpy(), acc_ref)
        assert_y_matches(L.y, y_ref, acc_ref)


@pytest.mark.parametrize("M", [1, 2, 16])
def test_layer_chain_on_caller_codes(M):
    """A chain layer given its input as codes (xq, scale, rowsum) equals forward_quantized."""
    K = 2048
    x, _ = activations(M, K, seed=5, dtype="bf16")
    xq, sc, rs = tb.quant_act(x)
    specs = [(K, 900), (K, 300)]
    layers, singles = [], []
    for i, (k, n) in enumerate(specs):
        packed, gamma = tb.pack_weights(dev(weights(n, k, seed=60 + i)))
        y = torch.empty((M, n), dtype=torch.bfloat16, device="cuda")
        acc = torch.empty((M, n), dtype=torch.int32, device="cuda")
        layers.append(tb.Layer(packed, gamma, None, y, xq=xq, scale=sc, rowsum=rs, acc_out=acc))
        singles.append(tb.forward_quantized(packed, gamma, xq, sc, rs, acc_out=True))
    tb.layer_chain(layers)
    for L, (y, a) in zip(layers, singles):
        assert torch.equal(L.acc_out, a) and torch.equal(L.y, y)


def test_layer_chain_matches_separate_forwards():
    K = 1024
    x, _ = activations(4, K, seed=1, dtype="bf16")
    specs = [(K, 700, x), (K, 900, x), (K, 300, None)]
    layers, singles = [], []
    for i, (k, n, xi) in enumerate(specs):
        packed, gamma = tb.pack_weights(dev(weights(n, k, seed=50 + i)))
        xi = xi if xi is not None else activations(4, k, seed=9, dtype="bf16")[0]
        layers.append(tb.Layer(packed, gamma, xi, torch.empty((4, n), dtype=torch.bfloat16, device="cuda")))
        singles.append(tb.forward(packed, gamma, xi))
    tb.layer_chain(layers)
    for L, y in zip(layers, singles):
        assert torch.equal(L.y, y)


def test_prepared_chain_equals_layer_chain():
    """A chain marshalled once (prepare_chain) and run twice gives layer_chain's outputs."""
    K = 1024
    x, _ = activations(4, K, seed=3, dtype="bf16")
    specs = [(K, 700, x), (K, 900, x), (K, 300, None)]
    layers, singles = [], []
    for i, (k, n, xi) in enumerate(specs):
        packed, gamma = tb.pack_weights(dev(weights(n, k, seed=90 + i)))
        xi = xi if xi is not None else activations(4, k, seed=11, dtype="bf16")[0]
        layers.append(tb.Layer(packed, gamma, xi, torch.empty((4, n), dtype=torch.bfloat16, device="cuda")))
        singles.append(tb.forward(packed, gamma, xi))
    plan = tb.prepare_chain(layers)
    for _ in range(2):
        for L in layers:
            L.y.zero_()
        plan.run()
        for L, y in zip(layers, singles):
            assert torch.equal(L.y, y)
    assert tb.device_status(plan.workspace) == tb.BL_OK


def test_shared_workspace_across_shapes_stays_consistent():
    """One workspace serves calls of different shapes in stream order."""
    shapes = [(1, 6912, 2560), (16, 300, 8640), (8, 3200, 8640), (3, 2560, 2560), (1, 6912, 2560)]
    ws = tb.new_workspace(max(tb.workspace_bytes(M, N, K) for M, N, K in shapes))
    for i, (M, N, K) in enumerate(shapes):
        packed, gamma = tb.pack_weights(dev(weights(N, K, seed=70 + i)))
        x, _ = activations(M, K, seed=80 + i, dtype="bf16")
        y1, a1 = tb.forward(packed, gamma, x, acc_out=True, workspace=ws)
        y2, a2 = tb.forward(packed, gamma, x, acc_out=True, workspace=tb.new_workspace(tb.workspace_bytes(M, N, K)))
        assert torch.equal(a1, a2) and torch.equal(y1, y2)
    assert int(ws[:256].count_nonzero().item()) == 0


# One token on caller codes with enough rows that no split is taken: units of
# 32 rows over stages of 2048 inputs.  Ragged N (not a multiple of 32), K with
# a partial last stage (down to a single 128-input block), and several layers
# of different K in one launch.
# Five to sixteen tokens on streamed codes (the mma path): groups with more
# units than resident blocks (units by ticket), units of one or two stages
# (shorter than the ring), ragged rows, K not a multiple of 1024 (a half-stage
# past K), absent tokens of a slot (9 and 13 of 16); codes given ("q") or
# quantised by the call ("x"); twice on one workspace.
MMA_GROUPS = [(8, [(512, 40000, "q")]), (16, [(1024, 30000, "q")]), (9, [(1536, 20000, "q"), (576, 7001, "x")]),
          (13, [(8192, 3000, "x"), (640, 9000, "q"), (2112, 1000, "x")]), (5, [(3200, 8640, "x")])]


@pytest.mark.parametrize("M,specs", MMA_GROUPS,
                         ids=["m%d-" % M + "+".join("%dx%d%s" % s for s in specs) for M, specs in MMA_GROUPS])
def test_mma_path_groups_match_the_oracle(M, specs):
    layers, refs = [], []
    for i, (K, N, given) in enumerate(specs):
        x, xf = activations(M, K, seed=400 + 7 * i + M, dtype="bf16")
        packed, gamma, T = oracle.pack_weights(weights(N, K, seed=410 + i))
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
        if given == "q":
            xq, sc, rs = tb.quant_act(x)
            layers.append(tb.Layer(dev(packed), dev(np.array([gamma], np.float32)), None, y, xq=xq, scale=sc,
                                   rowsum=rs, acc_out=acc))
        else:
            layers.append(tb.Layer(dev(packed), dev(np.array([gamma], np.float32)), x, y, acc_out=acc))
        refs.append(oracle.forward(T, gamma, xf))
    ws = tb.new_workspace(tb.chain_workspace_bytes(layers, M))
    for _ in range(2):
        tb.layer_chain(layers, workspace=ws)
        for L, (acc_ref, y_ref, *_) in zip(layers, refs):
            got = L.acc_out.cpu().numpy()
            assert np.array_equal(got, acc_ref), "acc differs at %s" % np.argwhere(got != acc_ref)[:5].tolist()
            assert_y_matches(L.y, y_ref, acc_ref)
    assert tb.device_status(ws) == tb.BL_OK


NARROW = [[(128, 6400)], [(1152, 6433)], [(8640, 7000)], [(2176, 3300), (4096, 3500), (128, 130)],
          [(14336, 3200), (8192, 3217)]]


@pytest.mark.parametrize("specs", NARROW, ids=lambda s: "+".join("%dx%d" % kn for kn in s))
def test_one_token_narrow_units_match_the_oracle(specs):
    layers, refs = [], []
    for i, (K, N) in enumerate(specs):
        x, xf = activations(1, K, seed=300 + i, dtype="bf16")
        xq, sc, rs = tb.quant_act(x)
        packed, gamma, T = oracle.pack_weights(weights(N, K, seed=310 + i))
        y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
        acc = torch.empty((1, N), dtype=torch.int32, device="cuda")
        layers.append(tb.Layer(dev(packed), dev(np.array([gamma], np.float32)), None, y, xq=xq, scale=sc,
                               rowsum=rs, acc_out=acc))
        refs.append(oracle.forward(T, gamma, xf))
    tb.layer_chain(layers)
    for L, (acc_ref, y_ref, *_) in zip(layers, refs):
        assert np.array_equal(L.acc_out.cpu().numpy(), acc_ref)
        assert_y_matches(L.y, y_ref, acc_ref)


# One token quantised by the quantisation kernel and streamed as codes in
# 32-row units: a single layer with too many inputs for the in-kernel staging
# and enough rows that no split is taken, and chains of several layers,
# distinct and shared inputs, K not a multiple of 2048 (and one not a multiple
# of 128, so the codes carry zero padding), fp32 and bf16 inputs, called twice
# on one workspace.
ONE_TOKEN_STREAMED = [(6400, 10240, "bf16"), (6464, 16448, "f32"), (7000, 28672, "bf16"), (6400, 12352, "bf16")]


@pytest.mark.parametrize("N,K,xdt", ONE_TOKEN_STREAMED)
def test_one_token_streamed_codes_match_the_oracle(N, K, xdt):
    x, xf = activations(1, K, seed=K + 3, dtype=xdt)
    packed, gamma, T = oracle.pack_weights(weights(N, K, seed=N + 5))
    ws = tb.new_workspace(tb.workspace_bytes(1, N, K))
    acc_ref, y_ref, *_ = oracle.forward(T, gamma, xf)
    for _ in range(2):
        y, acc = tb.forward(dev(packed), dev(np.array([gamma], np.float32)), x, acc_out=True, workspace=ws)
        assert np.array_equal(acc.cpu().numpy(), acc_ref)
        assert_y_matches(y, y_ref, acc_ref)
    assert tb.device_status(ws) == tb.BL_OK


@pytest.mark.parametrize("xdt", ["bf16", "f32"])
def test_one_token_chain_of_streamed_codes_matches_the_oracle(xdt):
    # (K, N, input): inputs a, a (shared), b, c; K = 8256 needs padding to 8320
    specs = [(8192, 3000, "a"), (8192, 2500, "a"), (8256, 1800, "b"), (3072, 900, "c")]
    xs = {}
    layers, refs = [], []
    for i, (K, N, name) in enumerate(specs):
        if name not in xs:
            xs[name] = activations(1, K, seed=200 + i, dtype=xdt)
        x, xf = xs[name]
        packed, gamma, T = oracle.pack_weights(weights(N, K, seed=210 + i))
        y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
        acc = torch.empty((1, N), dtype=torch.int32, device="cuda")
        layers.append(tb.Layer(dev(packed), dev(np.array([gamma], np.float32)), x, y, acc_out=acc))
        refs.append(oracle.forward(T, gamma, xf))
    ws = tb.new_workspace(tb.chain_workspace_bytes(layers, 1))
    for _ in range(2):
        tb.layer_chain(layers, workspace=ws)
        for L, (acc_ref, y_ref, *_) in zip(layers, refs):
            assert np.array_equal(L.acc_out.cpu().numpy(), acc_ref)
            assert_y_matches(L.y, y_ref, acc_ref)
    assert tb.device_status(ws) == tb.BL_OK


# One token quantised inside the decode kernel (small K, or one bf16 token of a
# single layer up to K = 9856) on 32-row units: ragged N and K, fp32 and bf16
# inputs and outputs; and a chain of such layers on different inputs.
NARROW_IN_KERNEL = [(6400, 2560, "bf16"), (6433, 1088, "f32"), (7000, 4096, "bf16"), (6464, 9856, "bf16"),
                    (6400, 64, "f32")]


@pytest.mark.parametrize("N,K,xdt", NARROW_IN_KERNEL)
def test_one_token_in_kernel_quantisation_narrow_units(N, K, xdt):
    _full_case(1, N, K, xdt, torch.float32 if xdt == "f32" else torch.bfloat16, tb.PATH_GEMV, seed=N + 3 * K)


def test_one_token_chain_in_kernel_quantisation_narrow_units():
    specs = [(2560, 3000), (2560, 2000), (1024, 1500)]
    layers, refs = [], []
    for i, (K, N) in enumerate(specs):
        x, xf = activations(1, K, seed=400 + i, dtype="bf16")
        packed, gamma, T = oracle.pack_weights(weights(N, K, seed=410 + i))
        layers.append(tb.Layer(dev(packed), dev(np.array([gamma], np.float32)), x,
                               torch.empty((1, N), dtype=torch.bfloat16, device="cuda"),
                               acc_out=torch.empty((1, N), dtype=torch.int32, device="cuda")))
        refs.append(oracle.forward(T, gamma, xf))
    tb.layer_chain(layers)
    for L, (acc_ref, y_ref, *_) in zip(layers, refs):
        assert np.array_equal(L.acc_out.cpu().numpy(), acc_ref)
        assert_y_matches(L.y, y_ref, acc_ref)
