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
