"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

Nothing here re-types the oracle's formulas.  Each test checks the oracle
against something independent of it: hand-worked examples under
``tests/golden/`` (each citing its passage), exact arithmetic (``math.fsum``,
``fractions``), library routines for special cases (integer and float64
matrix products), closed forms, invariants and statistics of the Gaussian
inputs the pages' workloads use.

Passages (web pages on BitNet b1.58):
  [AbsMean] "BitNet b1.58 and the 1-Bit AI Architecture Revolution",
            section "The BitLinear Layer and AbsMean Quantization".
  [Stack]   "BitNet's Real Bet: Designing the Whole Inference Stack",
            section "A low-bit model is a whole-stack design".
  [Energy]  "BitNet b1.58 and the 1-Bit AI Architecture Revolution",
            section "The Energy Revolution".
  [Norm]    "BitNet's Real Bet: Designing the Whole Inference Stack" (native
            training: RMSNorm, sub-layer normalisation) and "BitNet b1.58 and
            the 1-Bit AI Architecture Revolution", section "Empirical
            Performance and The New Scaling Law" (RMSNorm).
  [STE]     "BitNet b1.58 and the 1-Bit AI Architecture Revolution", section
            "Training Dynamics: The Straight-Through Estimator".
  [GLU]     "BitNet's Real Bet: Designing the Whole Inference Stack" (native
            training: SwiGLU, squared ReLU) and "A Two-Billion Ternary Bet"
            (squared-ReLU-style activations).
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth
from conftest import read_golden

EPS32 = np.float32(1e-5)


def ulp32(x) -> float:
    x = np.float32(x)
    return float(np.spacing(np.abs(x)))


# ----------------------------------------------------------------------------
# gamma = mean |W|  [AbsMean]
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("shape,seed", [((256, 256), 0), ((64, 2560), 1), ((691, 320), 2), ((8, 8640), 3)])
def test_gamma_matches_exact_mean(shape, seed):
    """gamma is the mean |W| rounded to fp32: compare with an exactly-rounded sum."""
    W = synth.latent_weights(*shape, seed=seed)
    g, total = oracle.absmean_gamma(W)
    exact_sum = math.fsum(np.abs(W.astype(np.float64)).ravel().tolist())
    ref = np.float32(exact_sum / W.size)
    assert abs(float(g) - float(ref)) <= ulp32(ref)
    # the double sum itself is within the sequential-summation error bound
    assert abs(total - exact_sum) <= W.size * 2.0 ** -52 * exact_sum


def test_gamma_exact_for_constant_magnitude():
    """|w| = c everywhere (random signs): every partial sum is an exact multiple of c."""
    rng = np.random.default_rng(5)
    for c in (np.float32(0.02), np.float32(0.0078125), np.float32(3.0)):
        W = (rng.choice([-1.0, 1.0], size=(37, 448)) * c).astype(np.float32)
        g, _ = oracle.absmean_gamma(W)
        assert g == c


def test_gamma_single_entry_and_zero():
    W = np.zeros((16, 64), dtype=np.float32)
    assert oracle.absmean_gamma(W)[0] == 0.0
    W[3, 17] = -0.75  # N*K = 1024 = 2^10, so the mean is exactly 0.75 / 1024
    assert oracle.absmean_gamma(W)[0] == np.float32(0.75 / 1024)


def test_gamma_uses_absolute_values_and_whole_matrix():
    """A mean of signed values, or of one row, would differ here."""
    W = np.array([[1.0, -1.0, 1.0, -1.0], [0.0, 0.0, 0.0, 4.0]], dtype=np.float32)
    assert oracle.absmean_gamma(W)[0] == np.float32(8.0 / 8)


# ----------------------------------------------------------------------------
# ternarisation  [AbsMean]
# ----------------------------------------------------------------------------

def _round_to_f32(fr: Fraction) -> Fraction:
    """Correctly rounded fp32 of an exact rational (ties to even), by bisection."""
    f = np.float32(float(fr))  # within one double rounding of fr
    best = None
    for cand in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        err = abs(Fraction(float(cand)) - fr)
        key = (err, int(np.frombuffer(np.float32(cand).tobytes(), np.uint32)[0]) & 1)
        if best is None or key < best[0]:
            best = (key, cand)
    return Fraction(float(best[1]))


def test_ternary_values_and_threshold_rule():
    """t in {-1,0,1}; t = 0 below half the scale, sign(w) above it (exact arithmetic)."""
    W = synth.latent_weights(96, 512, seed=11)
    g, _ = oracle.absmean_gamma(W)
    T = oracle.ternarize(W, g)
    assert set(np.unique(T).tolist()) <= {-1, 0, 1}
    d = Fraction(float(np.float32(g) + EPS32))  # the divisor gamma + eps as an fp32 number
    flat_w, flat_t = W.ravel(), T.ravel()
    for i in range(0, flat_w.size, 97):
        w = Fraction(float(flat_w[i]))
        r = _round_to_f32(w / d)  # the quotient as the fp32 division returns it
        if abs(r) < Fraction(1, 2):
            want = 0
        elif abs(r) > Fraction(1, 2):
            want = 1 if w > 0 else -1
        else:
            want = 0  # exactly one half: nearest even integer is 0
        assert flat_t[i] == want


def test_ternary_ties_go_to_even():
    """Quotients of exactly 0.5, 1.5 and 2.5: ties to even, then the clamp."""
    g = np.float32(0.25)
    d = np.float32(g + EPS32)
    half = np.float32(d * np.float32(0.5))
    assert float(half) * 2 == float(d)  # exact
    cases = [(half, 0), (-half, 0), (np.nextafter(half, np.float32(1)), 1),
             (np.nextafter(half, np.float32(0)), 0)]
    three_halves = np.float32(d * np.float32(1.5))
    if float(three_halves) == 1.5 * float(d):  # exact: rint(1.5) = 2, clamped to 1
        cases.append((three_halves, 1))
        cases.append((-three_halves, -1))
    W = np.array([[c for c, _ in cases]], dtype=np.float32)
    T = oracle.ternarize(W, g)
    assert T.ravel().tolist() == [t for _, t in cases]


def test_ternary_special_matrices():
    for c in (0.02, 1.0, 1e-3):
        W = np.full((4, 32), c, dtype=np.float32)
        g, _ = oracle.absmean_gamma(W)
        assert (oracle.ternarize(W, g) == 1).all()     # c / (c + 1e-5) rounds to 1
        assert (oracle.ternarize(-W, g) == -1).all()
    Z = np.zeros((4, 32), dtype=np.float32)
    g, _ = oracle.absmean_gamma(Z)
    assert g == 0 and (oracle.ternarize(Z, g) == 0).all()


def test_ternary_gaussian_statistics():
    """Gaussian latents: P(t = 0) = P(|Z| < E|Z| / 2) = erf(1 / (2 sqrt(pi)))."""
    W = synth.latent_weights(2560, 1728, seed=0)
    g, _ = oracle.absmean_gamma(W)
    T = oracle.ternarize(W, g)
    p0 = math.erf(1.0 / (2.0 * math.sqrt(math.pi)))  # 0.31002...
    assert abs((T == 0).mean() - p0) < 1e-3
    assert abs((T == 1).mean() - (1 - p0) / 2) < 1e-3
    assert abs((T == -1).mean() - (1 - p0) / 2) < 1e-3
    # gamma of N(0, s) latents is close to s * sqrt(2 / pi)
    assert abs(float(g) - 0.02 * math.sqrt(2 / math.pi)) < 2e-4


# ----------------------------------------------------------------------------
# packing  [Stack]
# ----------------------------------------------------------------------------

def test_pack_golden_layout():
    rows = read_golden("pack_layout.txt")
    pairs = [(rows[i][1], rows[i + 1][1]) for i in range(0, len(rows), 2)]
    for trow, brow in pairs:
        T = np.array([[int(v) for v in trow]], dtype=np.int8)
        want = np.array([int(b, 16) for b in brow], dtype=np.uint8)
        P = oracle.pack(T)
        assert P.ravel().tolist() == want.tolist()
        back, ok = oracle.unpack(P, T.shape[1])
        assert ok and (back == T).all()


def test_pack_round_trip_and_codes():
    rng = np.random.default_rng(3)
    T = rng.integers(-1, 2, size=(33, 640)).astype(np.int8)
    P = oracle.pack(T)
    assert P.shape == (33, 160)
    back, ok = oracle.unpack(P, 640)
    assert ok and (back == T).all()
    codes = np.stack([(P >> s) & 3 for s in (0, 2, 4, 6)])
    assert not (codes == 3).any()
    assert (oracle.pack(np.zeros((2, 64), np.int8)) == 0x55).all()
    bad = P.copy()
    bad[5, 7] |= 0xC0  # plant a code 3
    assert not oracle.unpack(bad, 640)[1]


def test_pack_counts_preserved():
    """Each byte holds four codes: the code histogram equals the ternary histogram."""
    rng = np.random.default_rng(4)
    T = rng.integers(-1, 2, size=(7, 256)).astype(np.int8)
    P = oracle.pack(T)
    codes = np.concatenate([((P >> s) & 3).ravel() for s in (0, 2, 4, 6)])
    for t in (-1, 0, 1):
        assert (codes == t + 1).sum() == (T == t).sum()


# ----------------------------------------------------------------------------
# per-token 8-bit activations  [Stack]
# ----------------------------------------------------------------------------

def test_act_quant_golden():
    rows = read_golden("act_quant.txt")
    for i in range(0, len(rows), 4):
        x = np.array([[float(v) for v in rows[i][1]]], dtype=np.float32)
        q, s, r = oracle.quant_act(x)
        assert q.ravel().tolist() == [int(v) for v in rows[i + 1][1]]
        assert s[0] == np.float32(rows[i + 2][1][0])
        assert r[0] == int(rows[i + 3][1][0])


def test_act_quant_invariants():
    x = synth.activations_f32(16, 3200, seed=7)
    q, s, r = oracle.quant_act(x)
    assert q.dtype == np.int8 and np.abs(q.astype(np.int32)).max() <= 127
    for m in range(x.shape[0]):
        j = int(np.argmax(np.abs(x[m])))
        assert q[m, j] == (127 if x[m, j] > 0 else -127)
        assert r[m] == int(q[m].astype(np.int64).sum())
        # rounding to nearest: |x - q/s| <= 1/(2s), up to fp32 rounding of x*s
        err = np.abs(x[m].astype(np.float64) - q[m] / np.float64(s[m]))
        assert err.max() <= (0.5 + 1e-5) / float(s[m])
        # monotone in x within the token
        order = np.argsort(x[m], kind="stable")
        assert (np.diff(q[m][order].astype(np.int32)) >= 0).all()
        # the scale maps the token's absmax to 127
        assert abs(float(s[m]) * float(np.abs(x[m]).max()) - 127) < 127 * 2 ** -22


def test_act_quant_zero_and_one_hot_tokens():
    x = np.zeros((3, 64), dtype=np.float32)
    x[1, 9] = -3.0
    x[2, 40] = 1e-7  # below the 1e-5 floor: scale saturates, codes stay small
    q, s, r = oracle.quant_act(x)
    assert (q[0] == 0).all() and r[0] == 0
    assert q[1, 9] == -127 and (np.delete(q[1], 9) == 0).all()
    assert abs(float(s[1]) - 127 / 3) <= ulp32(127 / 3)
    assert q[2, 40] == round(1e-7 * 127 / 1e-5)


# ----------------------------------------------------------------------------
# ternary x int8 product  [Energy]
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (3, 5, 64), (4, 8, 128), (2, 7, 48)])
def test_accumulate_matches_integer_matmul(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    q = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    T = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    acc = oracle.accumulate(q, T)
    assert (acc == q.astype(np.int64) @ T.astype(np.int64).T).all()


def test_accumulate_closed_forms():
    rng = np.random.default_rng(9)
    T = rng.integers(-1, 2, size=(12, 256)).astype(np.int8)
    q = np.zeros((1, 256), np.int8)
    q[0, 77] = 127
    assert (oracle.accumulate(q, T)[0] == 127 * T[:, 77].astype(np.int32)).all()
    q = rng.integers(-127, 128, size=(3, 256)).astype(np.int8)
    ones = np.ones((2, 256), np.int8)
    assert (oracle.accumulate(q, ones) == q.astype(np.int64).sum(1)[:, None]).all()
    assert (oracle.accumulate(q, -ones) == -q.astype(np.int64).sum(1)[:, None]).all()
    # extreme: |acc| = 127 * K stays exact
    big = np.full((1, 28672), -127, np.int8)
    assert oracle.accumulate(big, -np.ones((1, 28672), np.int8))[0, 0] == 127 * 28672


# ----------------------------------------------------------------------------
# dequantisation and the whole forward
# ----------------------------------------------------------------------------

def test_forward_golden():
    g = dict(read_golden("forward_small.txt"))
    W = np.array([[float(v) for v in g["W0"]], [float(v) for v in g["W1"]]], dtype=np.float32)
    x = np.array([[float(v) for v in g["x"]]], dtype=np.float32)
    packed, gamma, T = oracle.pack_weights(W)
    assert gamma == np.float32(g["gamma"][0])
    assert T[0].tolist() == [int(v) for v in g["T0"]]
    assert T[1].tolist() == [int(v) for v in g["T1"]]
    assert packed[0].tolist() == [int(b, 16) for b in g["packed0"]]
    assert packed[1].tolist() == [int(b, 16) for b in g["packed1"]]
    acc, y, q, s, r = oracle.forward(T, gamma, x)
    assert q[0].tolist() == [int(v) for v in g["q"]]
    assert s[0] == np.float32(g["s"][0])
    assert acc[0].tolist() == [int(v) for v in g["acc"]]
    assert y[0].tolist() == [float(v) for v in g["y"]]
    assert oracle.round_bf16(y)[0].tolist() == [int(b, 16) for b in g["y_bf16"]]


def test_bf16_rounding_golden():
    for expr, bits in read_golden("bf16_rounding.txt"):
        value = float(eval(expr, {"__builtins__": {}}))  # exact binary expressions
        assert oracle.round_bf16(np.array([value]))[0] == int(bits[0], 16), expr
    assert oracle.round_bf16(np.array([-0.0]))[0] == 0x8000


def test_round_f32_is_nearest():
    rng = np.random.default_rng(2)
    y = rng.standard_normal(1000) * 1e3
    f = oracle.round_f32(y)
    for v, r in zip(y[:200], f[:200]):
        lo, hi = np.nextafter(r, np.float32(-np.inf)), np.nextafter(r, np.float32(np.inf))
        assert abs(float(r) - v) <= abs(float(lo) - v) and abs(float(r) - v) <= abs(float(hi) - v)


def test_dequant_equals_dequantised_operands_product():
    """acc * gamma / s equals (q / s) @ (gamma * T)^T computed by float64 matmul."""
    W = synth.latent_weights(300, 512, seed=21)
    x = synth.activations_f32(5, 512, seed=22)
    _, gamma, T = oracle.pack_weights(W)
    acc, y, q, s, _ = oracle.forward(T, gamma, x)
    ref = (q.astype(np.float64) / s.astype(np.float64)[:, None]) @ (np.float64(gamma) * T.astype(np.float64)).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_forward_one_hot_closed_form():
    """One-hot x (value v at channel j): y[n] = t[n][j] * gamma * v up to fp32 rounding of s."""
    W = synth.latent_weights(64, 256, seed=31)
    _, gamma, T = oracle.pack_weights(W)
    for v, j in ((2.5, 3), (-0.37, 200), (40.0, 255)):
        x = np.zeros((1, 256), np.float32)
        x[0, j] = v
        acc, y, *_ = oracle.forward(T, gamma, x)
        want = T[:, j].astype(np.float64) * float(gamma) * float(np.float32(v))
        np.testing.assert_allclose(y[0], want, rtol=2.5e-7, atol=0)


def test_forward_power_of_two_equivariance():
    """Scaling a token by 2^k scales s by 2^-k exactly, so q is unchanged and y scales by 2^k."""
    W = synth.latent_weights(40, 320, seed=41)
    x = synth.activations_f32(3, 320, seed=42)
    _, gamma, T = oracle.pack_weights(W)
    acc1, y1, q1, *_ = oracle.forward(T, gamma, x)
    acc2, y2, q2, *_ = oracle.forward(T, gamma, (x * np.float32(8.0)).astype(np.float32))
    assert (q1 == q2).all() and (acc1 == acc2).all()
    np.testing.assert_array_equal(y2, y1 * 8.0)


def test_forward_approximates_full_precision_layer():
    """The W1.58A8 output tracks the full-precision x @ W^T (loose statistical pin)."""
    W = synth.latent_weights(512, 1024, seed=51)
    x = synth.activations_f32(4, 1024, seed=52, outliers=False)
    _, gamma, T = oracle.pack_weights(W)
    _, y, *_ = oracle.forward(T, gamma, x)
    full = x.astype(np.float64) @ W.astype(np.float64).T
    corr = np.corrcoef(y.ravel(), full.ravel())[0, 1]
    assert corr > 0.85


# ----------------------------------------------------------------------------
# RMSNorm before the activation quantisation  [Norm]
# ----------------------------------------------------------------------------

def _golden_rmsnorm_cases():
    rows = read_golden("rmsnorm.txt")
    for i in range(0, len(rows), 5):
        (kx, x), (kg, g), (ke, e), (kv, v), (ku, u) = rows[i:i + 5]
        assert (kx, kg, ke, kv, ku) == ("x", "g", "eps", "v", "ulps")
        yield ([float(t) for t in x], None if g == ["-"] else [float(t) for t in g], float(e[0]),
               [float(t) for t in v], int(u[0]))


def test_rmsnorm_golden_cases():
    n = 0
    for x, g, eps, v, ulps in _golden_rmsnorm_cases():
        got = oracle.rmsnorm(np.array([x], np.float32), None if g is None else np.array(g, np.float32), eps, False)[0]
        for a, b in zip(got, v):
            assert abs(float(a) - b) <= ulps * max(ulp32(b), 1e-45), (x, g, eps, got, v)
        n += 1
    assert n == 6


@pytest.mark.parametrize("K,seed", [(2560, 0), (64, 1), (8640, 2)])
def test_rmsnorm_output_has_unit_rms(K, seed):
    """With eps = 0 and no gain the output's mean square is 1 (fp32 rounding only)."""
    _, x = synth.activations_bf16(4, K, seed=seed)
    v = oracle.rmsnorm(x, None, 0.0, False)
    for row in v.astype(np.float64):
        ms = math.fsum(float(t) * float(t) for t in row) / K
        assert abs(ms - 1.0) < 4e-7


def test_rmsnorm_power_of_two_scaling_and_gain():
    """Scaling x by 2^j leaves the output unchanged; a gain of 2^j scales it exactly."""
    _, x = synth.activations_bf16(3, 512, seed=5)
    base = oracle.rmsnorm(x, None, 0.0, False)
    for j in (-3, 1, 7):
        assert np.array_equal(oracle.rmsnorm(x * np.float32(2.0 ** j), None, 0.0, False), base)
        g = np.full(512, 2.0 ** j, np.float32)
        assert np.array_equal(oracle.rmsnorm(x, g, 0.0, False), base * np.float32(2.0 ** j))


def _bf16_rne_bits(f: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 round-to-nearest-even, on the bit patterns (finite inputs)."""
    u = f.astype(np.float32).view(np.uint32).astype(np.uint64)
    lower = u & 0xFFFF
    upper = u >> 16
    round_up = (lower > 0x8000) | ((lower == 0x8000) & ((upper & 1) == 1))
    return (upper + round_up.astype(np.uint64)).astype(np.uint16)


def test_rmsnorm_bf16_output_is_the_rounded_fp32_output():
    _, x = synth.activations_bf16(5, 2560, seed=6)
    g = synth.activations_bf16(1, 2560, seed=7)[1][0]
    f32 = oracle.rmsnorm(x, g, 1e-6, False)
    b16 = oracle.rmsnorm(x, g, 1e-6, True)
    want = (_bf16_rne_bits(f32).astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(b16, want)


def test_rmsnorm_quant_of_a_zero_token():
    v, q, s, r = oracle.rmsnorm_quant(np.zeros((1, 64), np.float32), None, 1e-6, True)
    assert not v.any() and not q.any() and r[0] == 0 and s[0] == np.float32(127.0) / EPS32


# ----------------------------------------------------------------------------
# The FFN's gated activation before the down BitLinear  [GLU]
# ----------------------------------------------------------------------------

def test_glu_golden_cases():
    rows = read_golden("glu.txt")
    n = 0
    for i in range(0, len(rows), 5):
        (ka, a), (kg, g), (ku, u), (kh, h), (kl, ul) = rows[i:i + 5]
        assert (ka, kg, ku, kh, kl) == ("act", "gate", "up", "h", "ulps")
        act = {"relu2": oracle.GLU_RELU2, "silu": oracle.GLU_SILU}[a[0]]
        got = oracle.glu(np.array([[float(t) for t in g]], np.float32), np.array([[float(t) for t in u]], np.float32),
                         act, False)[0]
        for x, want in zip(got, (float(t) for t in h)):
            assert abs(float(x) - want) <= int(ul[0]) * max(ulp32(want), 1e-45), (a, got, h)
        n += 1
    assert n == 3


def test_silu_odd_part_is_the_identity():
    """silu(z) - silu(-z) = z * (sigma(z) + sigma(-z)) = z."""
    z = synth.activations_f32(1, 4096, seed=21)[0] * np.float32(3.0)
    one = np.ones_like(z)
    d = oracle.glu(z[None], one[None], oracle.GLU_SILU, False)[0].astype(np.float64) - \
        oracle.glu(-z[None], one[None], oracle.GLU_SILU, False)[0].astype(np.float64)
    tol = np.array([ulp32(t) for t in z]) * 2
    assert (np.abs(d - z.astype(np.float64)) <= tol).all()


def test_silu_limits():
    """Far right silu(z) = z in fp32; far left it is z * e^z to first order."""
    one = np.ones((1, 2), np.float32)
    hi = oracle.glu(np.array([[30.0, 60.0]], np.float32), one, oracle.GLU_SILU, False)[0]
    assert hi[0] == np.float32(30.0) and hi[1] == np.float32(60.0)
    lo = oracle.glu(np.array([[-30.0, -60.0]], np.float32), one, oracle.GLU_SILU, False)[0]
    for z, v in zip((-30.0, -60.0), lo):
        assert abs(float(v) - z * math.exp(z)) <= 1e-6 * abs(z * math.exp(z))


def test_relu2_scales_by_powers_of_four():
    g = synth.activations_f32(2, 512, seed=22)
    u = synth.activations_f32(2, 512, seed=23)
    base = oracle.glu(g, u, oracle.GLU_RELU2, False)
    for j in (-2, 3):
        got = oracle.glu(g * np.float32(2.0 ** j), u, oracle.GLU_RELU2, False)
        assert np.array_equal(got, base * np.float32(4.0 ** j))
    assert (base[g <= 0] == 0).all()


def test_glu_bf16_output_rounds_the_relu2_product():
    g = synth.activations_f32(3, 2048, seed=24)
    u = synth.activations_f32(3, 2048, seed=25)
    f32 = oracle.glu(g, u, oracle.GLU_RELU2, False)
    b16 = oracle.glu(g, u, oracle.GLU_RELU2, True)
    assert np.array_equal(b16, (_bf16_rne_bits(f32).astype(np.uint32) << 16).view(np.float32))


# ----------------------------------------------------------------------------
# The straight-through backward  [STE]
# ----------------------------------------------------------------------------

def _ste_case(M, N, K, seed):
    W = synth.latent_weights(N, K, seed=seed)
    _, gamma, T = oracle.pack_weights(W)
    _, x = synth.activations_bf16(M, K, seed=seed + 1)
    q, s, _ = oracle.quant_act(x)
    dy = synth.activations_f32(M, N, seed=seed + 2)
    return T, gamma, q, s, dy


@pytest.mark.parametrize("M,N,K,seed", [(4, 48, 64, 0), (16, 96, 128, 1), (7, 33, 256, 2)])
def test_ste_grads_match_float64_products(M, N, K, seed):
    """dx = gamma (dy . t) and dW = dy^T . xhat, against numpy's float64 products."""
    T, gamma, q, s, dy = _ste_case(M, N, K, seed)
    dx = oracle.ste_grad_input(dy, T, gamma)
    want = float(gamma) * (dy.astype(np.float64) @ T.astype(np.float64))
    assert np.allclose(dx, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    xhat = oracle.ste_xhat(q, s)
    dw = oracle.ste_grad_weight(dy, xhat)
    want = dy.astype(np.float64).T @ xhat.astype(np.float64)
    assert np.allclose(dw, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_ste_one_hot_gradients_select_rows():
    """A one-hot dy picks one row of gamma * t for dx and one token of xhat for dW."""
    T, gamma, q, s, dy = _ste_case(3, 20, 64, 3)
    dy = np.zeros_like(dy)
    dy[1, 7] = 1.0
    dx = oracle.ste_grad_input(dy, T, gamma)
    assert np.array_equal(dx[1], float(gamma) * T[7].astype(np.float64)) and not dx[0].any() and not dx[2].any()
    xhat = oracle.ste_xhat(q, s)
    dw = oracle.ste_grad_weight(dy, xhat)
    assert np.array_equal(dw[7], xhat[1].astype(np.float64)) and not np.delete(dw, 7, axis=0).any()


def test_ste_xhat_is_the_bf16_rounding_of_q_over_s():
    T, gamma, q, s, dy = _ste_case(5, 8, 256, 4)
    xhat = oracle.ste_xhat(q, s)
    f32 = (q.astype(np.float32) / s[:, None]).astype(np.float32)
    assert np.array_equal(xhat, (_bf16_rne_bits(f32).astype(np.uint32) << 16).view(np.float32))


def test_ste_grads_share_the_bilinear_form():
    """<dx, xhat> = <dW, gamma t> = <dy, xhat . (gamma t)^T> (Euler's identity for a bilinear form)."""
    T, gamma, q, s, dy = _ste_case(6, 40, 128, 5)
    xhat = oracle.ste_xhat(q, s)
    dx = oracle.ste_grad_input(dy, T, gamma)
    dw = oracle.ste_grad_weight(dy, xhat)
    a = math.fsum((dx * xhat.astype(np.float64)).ravel())
    b = math.fsum((dw * (float(gamma) * T.astype(np.float64))).ravel())
    y = xhat.astype(np.float64) @ (float(gamma) * T.astype(np.float64)).T
    c = math.fsum((dy.astype(np.float64) * y).ravel())
    scale = math.fsum(np.abs(dy.astype(np.float64) * y).ravel())
    assert abs(a - c) <= 1e-12 * scale and abs(b - c) <= 1e-12 * scale
