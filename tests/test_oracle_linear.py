"""Pins for the oracle's contraction, dequantisation, epilogues and the two FFN
compositions.

Sources: nnterp encyclopedia "bitnet": "The projections quantize their inputs
and weights" (the output equals the linear map of the rounded input by the
ternarised weight exactly), "The block, in order" (out = h + down(ffn_sub_norm(
relu(gate(z))^2 * up(z)))), "The MLP gates with a squared ReLU", "Scaling inside
a sublayer is undone by the sub-norm"; "bitnetv2-model" README, "Architecture
Overview" (512 -> 2048 -> 512 H-BitLinear FFN, silu).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests.exact import nearest_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_golden_linear_example():
    ex = _load("linear_example.json")
    q = np.array(ex["q"], dtype=np.int8)
    t = np.array(ex["t"], dtype=np.int8)
    acc = oracle.contract(q, t)
    np.testing.assert_array_equal(acc, np.array(ex["acc"], dtype=np.int32))
    y = oracle.dequant(acc, np.array([ex["s"]], dtype=np.float32), ex["gamma"])
    for n, (num, den) in enumerate(ex["y_rational"][0]):
        assert y[0, n] == nearest_f32(Fraction(num, den))


@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 5, 16), (8, 8, 64), (17, 9, 100)])
def test_contract_brute_force_int64(shape):
    """Library routine: an int64 matmul of the codes."""
    M, N, K = shape
    rng = np.random.default_rng(M * 100 + N)
    q = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    t = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    want = q.astype(np.int64) @ t.astype(np.int64).T
    np.testing.assert_array_equal(oracle.contract(q, t), want.astype(np.int32))


def test_contract_extremes_and_invariants():
    K = 16384
    q = np.full((2, K), 127, dtype=np.int8)
    q[1] = -128
    t = np.ones((2, K), dtype=np.int8)
    t[1] = -1
    acc = oracle.contract(q, t)
    assert acc[0, 0] == 127 * K and acc[1, 1] == 128 * K and acc[0, 1] == -127 * K
    rng = np.random.default_rng(12)
    q = rng.integers(-127, 128, size=(4, 96)).astype(np.int8)
    t = rng.integers(-1, 2, size=(6, 96)).astype(np.int8)
    perm = rng.permutation(96)
    np.testing.assert_array_equal(oracle.contract(q[:, perm], t[:, perm]), oracle.contract(q, t))
    np.testing.assert_array_equal(oracle.contract(-q, t), -oracle.contract(q, t))


def test_dequant_exactly_rounded():
    """y = acc * gamma / s, rounded once from the exact rational."""
    rng = np.random.default_rng(13)
    acc = rng.integers(-300000, 300000, size=(4, 7)).astype(np.int32)
    s = rng.uniform(0.5, 200, 4).astype(np.float32)
    g = np.float32(0.0173)
    y = oracle.dequant(acc, s, g)
    for (m, n), a in np.ndenumerate(acc):
        exact = Fraction(int(a)) * Fraction(float(g)) / Fraction(float(s[m]))
        want = nearest_f32(exact)
        if y[m, n] != want:       # fp64 double rounding can only matter next to a midpoint
            assert abs(Fraction(float(y[m, n])) - exact) <= Fraction(float(np.spacing(want))) * Fraction(1, 2) * (1 + Fraction(1, 10**8))
    assert np.all(oracle.dequant(np.zeros((2, 3), np.int32), s[:2], g) == 0)


def test_bitlinear_is_the_dense_map_of_dequantised_operands():
    """y equals (q/s) @ (gamma * t)^T in fp64, to fp32 rounding."""
    rng = np.random.default_rng(14)
    M, K, N = 8, 256, 512
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    X = rng.standard_normal((M, K)).astype(np.float32)
    g, t, _ = oracle.quantize_weights(W)
    y = oracle.bitlinear(X, t, g)
    q, s, _ = oracle.quant_act(X)
    dense = (q.astype(np.float64) / s[:, None].astype(np.float64)) @ (float(g) * t.astype(np.float64)).T
    # exact zeros of the integer map come out of the fp64 product as ~1e-16
    np.testing.assert_allclose(y, dense, rtol=1.2e-7, atol=1e-12)
    assert np.all(y[oracle.contract(q, t) == 0] == 0)


def test_bitlinear_homogeneity():
    """BitLinear(2^k x) = 2^k BitLinear(x) bit-exactly with no prelude."""
    rng = np.random.default_rng(15)
    W = (rng.standard_normal((64, 128)) * 0.02).astype(np.float32)
    X = rng.standard_normal((4, 128)).astype(np.float32)
    g, t, _ = oracle.quantize_weights(W)
    y = oracle.bitlinear(X, t, g)
    for k in (-2, 3):
        np.testing.assert_array_equal(oracle.bitlinear(X * np.float32(2.0 ** k), t, g),
                                      y * np.float32(2.0 ** k))


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(16)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 100,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.005859375, 3.0e38, 1e-40],
                                 dtype=np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(x), want)


def test_golden_relu2_and_silu():
    ex = _load("ffn_examples.json")
    r = ex["relu2_glu"]
    m = oracle.relu2_glu(np.array(r["g"], np.float32), np.array(r["u"], np.float32))
    np.testing.assert_array_equal(m, np.array(r["m"], np.float32))
    assert oracle.silu(np.array(ex["silu"]["y"], np.float32))[0] == 0.0


def test_silu_against_fp64_closed_form():
    ys = np.array([-100.0, -20.0, -1.5, -1e-3, 0.25, 1.0, 3.0, 50.0, 1e4], dtype=np.float32)
    got = oracle.silu(ys)
    for y, v in zip(ys, got):
        d = float(y)
        assert v == np.float32(d / (1.0 + math.exp(-d))) or abs(v - d / (1 + math.exp(-d))) <= abs(v) * 6e-8


# ---- SiLU pinned by the mathematics of y * sigmoid(y), not by its formula

def _f(v):
    return Fraction(float(v))


def test_silu_odd_part_is_the_identity():
    """silu(y) - silu(-y) = y for every y (sigmoid(y) + sigmoid(-y) = 1), up to
    the two fp32 roundings of the oracle's outputs; checked in exact rationals.
    A wrong factor or an added term breaks it."""
    ys = np.concatenate([np.linspace(-30, 30, 6001), np.geomspace(1e-6, 80, 400)]).astype(np.float32)
    pos, neg = oracle.silu(ys), oracle.silu(-ys)
    for y, a, b in zip(ys, pos, neg):
        half = (_f(np.spacing(np.abs(a))) + _f(np.spacing(np.abs(b)))) / 2
        assert abs(_f(a) - _f(b) - _f(y)) <= half, (y, a, b)


def test_silu_even_part_is_y_tanh_half_y():
    """silu(y) + silu(-y) = y (sigmoid(y) - sigmoid(-y)) = y tanh(y / 2).  This
    separates y * sigmoid(y) from y * sigmoid(-y) (an exp(+y) sign slip, which
    has the same odd part but the opposite even part)."""
    ys = np.linspace(-12, 12, 2401).astype(np.float32)
    got = oracle.silu(ys).astype(np.float64) + oracle.silu(-ys).astype(np.float64)
    want = np.array([float(y) * math.tanh(float(y) / 2) for y in ys])
    tol = 2 * np.spacing(np.abs(oracle.silu(np.abs(ys)))).astype(np.float64) + 1e-300
    assert np.all(np.abs(got - want) <= tol)
    assert np.all(got[ys != 0] > 0)          # y tanh(y/2) > 0 away from 0


def test_silu_limits():
    """y >> 0: sigmoid(y) = 1 to fp32 precision, silu(y) == y.  y << 0:
    silu(y) = y e^y (1 - e^y + ...) -> 0 from below.  y -> 0: silu(y) / y -> 1/2."""
    big = np.linspace(20, 80, 61).astype(np.float32)
    np.testing.assert_array_equal(oracle.silu(big), big)
    for y in (-20.0, -30.0, -50.0, -80.0):
        v = float(oracle.silu(np.array([y], np.float32))[0])
        assert v < 0
        assert abs(v / (y * math.exp(y)) - 1) <= 1e-6
    for y in (1e-4, -1e-4, 1e-6):
        v = float(oracle.silu(np.array([y], np.float32))[0])
        assert abs(v / float(np.float32(y)) - 0.5) <= 1e-4


def test_silu_minimum_is_at_minus_one_minus_lambert_w():
    """silu has one minimum: silu'(y) = 0 gives (1 + y) e^-y = -1, so
    y* = -1 - W(1/e) = -1.27846454... and silu(y*) = 1 + y* = -W(1/e)
    (W = Lambert's W function, principal branch)."""
    from scipy.special import lambertw
    w = float(lambertw(1.0 / math.e).real)
    y_star = -1.0 - w
    ys = np.linspace(-1.6, -1.0, 60001).astype(np.float32)
    v = oracle.silu(ys).astype(np.float64)
    i = int(np.argmin(v))
    assert abs(float(ys[i]) - y_star) <= 2e-3   # the minimum is flat: v - min ~ (y - y*)^2
    assert abs(v[i] - (-w)) <= 2.0 ** -24 * w
    assert np.all(np.diff(v[: i + 1]) <= 1e-7) and np.all(np.diff(v[i:]) >= -1e-7)


# ---- H-BitLinear pinned through a Sylvester Hadamard weight

def _sylvester(n):
    from scipy.linalg import hadamard
    return hadamard(n).astype(np.int8)


def _x_with_exact_transform(n, seed, e=-3):
    """x = (H v / sqrt(n)) 2^e for an integer v with max|v| = 127, n a power of
    four (sqrt(n) a power of two): x is exact in fp32 and its normalised
    transform is exactly v 2^e, so per-token quantisation returns v itself."""
    rng = np.random.default_rng(seed)
    v = rng.integers(-127, 128, size=n).astype(np.int64)
    v[rng.integers(n)] = 127 * (1 if rng.random() < 0.5 else -1)
    H = _sylvester(n).astype(np.int64)
    x = (H @ v).astype(np.float64) / math.sqrt(n) * 2.0 ** e
    assert np.all(np.float32(x) == x)
    return x.astype(np.float32)[None, :], v


@pytest.mark.parametrize("n", [16, 64, 256])
def test_hbitlinear_with_a_hadamard_weight_returns_sqrt_n_x(n):
    """An H-BitLinear whose ternary weight is the Sylvester matrix H (entries
    +-1, so gamma = mean|W| = 1) computes H . dequant(quant(H x / sqrt(n))).
    Since H H^T = n I that is sqrt(n) x, exactly when the quantiser's rounding
    is exact (x built so that H x / sqrt(n) is an integer vector times 2^e)."""
    H = _sylvester(n)
    W = H.astype(np.float32) * np.float32(0.75)      # any |W| = c gives gamma = c, t = H
    g, T, _ = oracle.quantize_weights(W)
    assert g == np.float32(0.75)
    np.testing.assert_array_equal(T, H)
    x, v = _x_with_exact_transform(n, seed=n)
    q, s, _ = oracle.quant_act(x, oracle.PRELUDE_FWHT)
    np.testing.assert_array_equal(q[0].astype(np.int64), v)
    y = oracle.bitlinear(x, T, np.float32(1.0), oracle.PRELUDE_FWHT)
    np.testing.assert_array_equal(y, (np.float32(math.sqrt(n)) * x).astype(np.float32))
    y = oracle.bitlinear(x, T, g, oracle.PRELUDE_FWHT)        # gamma scales the output
    np.testing.assert_array_equal(y, (np.float32(0.75 * math.sqrt(n)) * x).astype(np.float32))


@pytest.mark.parametrize("n", [64, 256])
def test_hffn_with_hadamard_weights(n):
    """The H-FFN W2 . silu(W1 . x) with both weights the Sylvester matrix
    (gamma = 1): the first H-BitLinear returns sqrt(n) x exactly (previous
    test), so the hidden activation is silu(sqrt(n) x); the second returns
    H q / s with q / s the int8 rounding of H h / sqrt(n), i.e. sqrt(n) h plus
    H e with |e| <= 1 / (2 s) per element: |out - sqrt(n) h| <= n / (2 s) +
    fp32 error.  A dropped transform, a transposed stage order or a missing
    activation breaks one of the two."""
    H = _sylvester(n)
    x, _ = _x_with_exact_transform(n, seed=3 * n, e=-5)
    out, h = oracle.hffn(x, H, np.float32(1.0), H, np.float32(1.0), keep=True)
    y1 = (np.float32(math.sqrt(n)) * x).astype(np.float32)
    np.testing.assert_array_equal(h, oracle.silu(y1))
    _, s2, _ = oracle.quant_act(h, oracle.PRELUDE_FWHT)
    err = np.abs(out.astype(np.float64) - math.sqrt(n) * h.astype(np.float64))
    bound = n / (2.0 * float(s2[0])) + 1e-5 * math.sqrt(n) * np.abs(h).max()
    assert np.all(err <= bound), (err.max(), bound)
    # and it is a real transform of h, not h itself: without the second
    # Hadamard prelude the result would be H h, far from sqrt(n) h
    assert np.abs(H.astype(np.float64) @ h[0] - math.sqrt(n) * h[0]).max() > 10 * bound


def _ffn_case(M=6, H=64, I=128, seed=17):
    rng = np.random.default_rng(seed)
    Wg = (rng.standard_normal((I, H)) * 0.02).astype(np.float32)
    Wu = (rng.standard_normal((I, H)) * 0.02).astype(np.float32)
    Wd = (rng.standard_normal((H, I)) * 0.02).astype(np.float32)
    x = rng.standard_normal((M, H)).astype(np.float32)
    gg, Tg, _ = oracle.quantize_weights(Wg)
    gu, Tu, _ = oracle.quantize_weights(Wu)
    gd, Td, _ = oracle.quantize_weights(Wd)
    return x, (Tg, gg, Tu, gu, Td, gd)


def test_ffn_matches_its_written_out_steps():
    """The composition equals the block order written out with pinned parts."""
    x, (Tg, gg, Tu, gu, Td, gd) = _ffn_case()
    out, m, qm, sm = oracle.ffn_relu2(x, Tg, gg, Tu, gu, Td, gd, keep=True)
    G = oracle.bitlinear(x, Tg, gg, oracle.PRELUDE_RMSNORM, eps=1e-5)
    U = oracle.bitlinear(x, Tu, gu, oracle.PRELUDE_RMSNORM, eps=1e-5)
    m2 = oracle.relu2_glu(G, U)
    np.testing.assert_array_equal(m, m2)
    D = oracle.bitlinear(m2, Td, gd, oracle.PRELUDE_RMSNORM, eps=1e-5)
    np.testing.assert_array_equal(out, (x + D).astype(np.float32))


def test_ffn_relu2_zero_where_gate_nonpositive():
    x, (Tg, gg, Tu, gu, Td, gd) = _ffn_case(seed=18)
    _, m, _, _ = oracle.ffn_relu2(x, Tg, gg, Tu, gu, Td, gd, keep=True)
    G = oracle.bitlinear(x, Tg, gg, oracle.PRELUDE_RMSNORM, eps=1e-5)
    assert np.all(m[G <= 0] == 0)
    assert np.any(G <= 0) and np.any(m != 0)


def test_ffn_residual_identity():
    """out - x equals the no-residual variant exactly (fp32, before any bf16 cast)."""
    x, w = _ffn_case(seed=19)
    with_res = oracle.ffn_relu2(x, *w, residual=True)
    no_res = oracle.ffn_relu2(x, *w, residual=False)
    np.testing.assert_array_equal(with_res, (x + no_res).astype(np.float32))


def test_ffn_sub_norm_scale_invariance():
    """Scaling m by 2 leaves the down projection unchanged: bit-identical with
    eps = 0 (the sub-norm undoes a scaling of its input)."""
    x, (Tg, gg, Tu, gu, Td, gd) = _ffn_case(seed=20)
    _, m, _, _ = oracle.ffn_relu2(x, Tg, gg, Tu, gu, Td, gd, keep=True)
    a = oracle.bitlinear(m, Td, gd, oracle.PRELUDE_RMSNORM, eps=0.0)
    b = oracle.bitlinear(m * np.float32(2.0), Td, gd, oracle.PRELUDE_RMSNORM, eps=0.0)
    np.testing.assert_array_equal(a, b)


def test_hffn_matches_its_written_out_steps():
    rng = np.random.default_rng(22)
    M, D, F = 5, 64, 256
    W1 = (rng.standard_normal((F, D)) * 0.02).astype(np.float32)
    W2 = (rng.standard_normal((D, F)) * 0.02).astype(np.float32)
    X = rng.standard_normal((M, D)).astype(np.float32)
    g1, T1, _ = oracle.quantize_weights(W1)
    g2, T2, _ = oracle.quantize_weights(W2)
    out, h = oracle.hffn(X, T1, g1, T2, g2, keep=True)
    # written out: FWHT -> quant -> contract -> dequant -> silu -> FWHT -> ...
    q1, s1, _ = oracle.quant_act(oracle.fwht(X))
    Y1 = oracle.dequant(oracle.contract(q1, T1), s1, g1)
    H = oracle.silu(Y1)
    np.testing.assert_array_equal(h, H)
    q2, s2, _ = oracle.quant_act(oracle.fwht(H))
    np.testing.assert_array_equal(out, oracle.dequant(oracle.contract(q2, T2), s2, g2))


# ---- the block after attention: o_proj with attn_sub_norm, residual, FFN

def _tail_case(M=5, H=64, I=128, seed=31):
    rng = np.random.default_rng(seed)
    Ws = {k: (rng.standard_normal(shape) * 0.02).astype(np.float32)
          for k, shape in (("Wo", (H, H)), ("Wg", (I, H)), ("Wu", (I, H)), ("Wd", (H, I)))}
    q = {k: oracle.quantize_weights(W) for k, W in Ws.items()}
    a = rng.standard_normal((M, H)).astype(np.float32)
    x = rng.standard_normal((M, H)).astype(np.float32)
    w = (q["Wo"][1], q["Wo"][0], q["Wg"][1], q["Wg"][0], q["Wu"][1], q["Wu"][0], q["Wd"][1],
         q["Wd"][0])
    gains = dict(attn_gain=rng.uniform(0.5, 1.5, H).astype(np.float32),
                 post_gain=rng.uniform(0.5, 1.5, H).astype(np.float32),
                 sub_gain=rng.uniform(0.5, 1.5, I).astype(np.float32))
    return a, x, w, gains


def test_block_tail_attn_sub_norm_undoes_scaling():
    """nnterp "bitnet", "Scaling inside a sublayer is undone by the sub-norm":
    scaling the attention output a by 2^k leaves the block's output bit for
    bit unchanged when eps = 0 (RMSNorm(2^k a) = RMSNorm(a) exactly)."""
    a, x, w, gains = _tail_case()
    base = oracle.block_tail(a, x, *w, eps=0.0, **gains)
    for k in (-3, 1, 5):
        np.testing.assert_array_equal(
            oracle.block_tail(a * np.float32(2.0 ** k), x, *w, eps=0.0, **gains), base)


def test_block_tail_reduces_to_the_ffn_when_o_proj_is_zero():
    """All-zero o_proj weights (gamma 0, every code 0) give o = 0 exactly, so
    h = x and the block is the pinned FFN of x."""
    a, x, w, gains = _tail_case(seed=32)
    To0 = np.zeros_like(w[0])
    got = oracle.block_tail(a, x, To0, np.float32(0.0), *w[2:], **gains)
    want = oracle.ffn_relu2(x, *w[2:], pre_gain=gains["post_gain"], sub_gain=gains["sub_gain"])
    np.testing.assert_array_equal(got, want)


def test_block_tail_reduces_to_o_proj_when_the_ffn_is_zero():
    """All-zero gate/up weights give m = 0, whose sub-norm codes are 0 (zero
    row: q = 0, s = 1), so the FFN adds exactly 0 and the block is
    x + BitLinear(RMSNorm(a)) (the pinned BitLinear with a residual)."""
    a, x, w, gains = _tail_case(seed=33)
    Z = np.zeros_like(w[2])
    got, h = oracle.block_tail(a, x, w[0], w[1], Z, np.float32(0.0), Z, np.float32(0.0), w[6],
                               w[7], keep=True, **gains)
    want = oracle.bitlinear(a, w[0], w[1], oracle.PRELUDE_RMSNORM, gain=gains["attn_gain"],
                            residual=x)
    np.testing.assert_array_equal(h, want)
    np.testing.assert_array_equal(got, want)



def test_block_tail_ffn_residual_is_h():
    """The FFN's residual is h (the stream after the attention residual), not
    x: out = fl32(h + FFN_without_residual(h)) bit for bit."""
    a, x, w, gains = _tail_case(seed=34)
    out, h = oracle.block_tail(a, x, *w, keep=True, **gains)
    d = oracle.ffn_relu2(h, *w[2:], pre_gain=gains["post_gain"], sub_gain=gains["sub_gain"],
                         residual=False)
    np.testing.assert_array_equal(out, (h + d).astype(np.float32))
    assert not np.array_equal(out, (x + d).astype(np.float32))
