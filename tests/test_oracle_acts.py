"""Pins for the oracle's activation side: per-token int8 absmax quant, the
RMSNorm prelude and the normalised fast Walsh-Hadamard transform.

Sources: nnterp encyclopedia "bitnet", "The projections quantize their inputs
and weights" (per token, 255 levels, round(x * 127 / max|x|)), "The block, in
order" and "Config" (RMSNorm, eps 1e-5), "Scaling inside a sublayer is undone
by the sub-norm"; "bitnetv2-model" README, "Special Features" (Hadamard
transform on power-of-two widths).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg

import oracle
from tests.exact import f32_div, f32_mul, nearest_f32, rint_half_even

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------- quant

def test_golden_quant_examples():
    for case in _load("quant_examples.json")["cases"]:
        x = np.array([case["x"]], dtype=np.float32)
        q, s, rs = oracle.quant_act(x)
        np.testing.assert_array_equal(q[0], np.array(case["q"], dtype=np.int8), err_msg=case["note"])
        if "s" in case:
            assert s[0] == np.float32(case["s"]), case["note"]
        else:
            num, den = case["s_rational"]
            assert s[0] == nearest_f32(Fraction(num, den)), case["note"]
        assert rs[0] == case["rowsum"]


def test_quant_closed_forms():
    # one-hot rows map the hot element to +-127 exactly
    rng = np.random.default_rng(1)
    for _ in range(200):
        K = int(rng.integers(1, 300))
        x = np.zeros((1, K), dtype=np.float32)
        k = int(rng.integers(0, K))
        x[0, k] = np.float32(rng.standard_normal() * 10 ** rng.uniform(-20, 20))
        q, s, _ = oracle.quant_act(x)
        assert q[0, k] == (127 if x[0, k] > 0 else -127)
        assert np.count_nonzero(q) == 1
    # a constant row maps to all +-127
    for c in (1.0, -3.5, 1e-30, 7e30):
        q, _, rs = oracle.quant_act(np.full((1, 64), c, dtype=np.float32))
        assert np.all(q == (127 if c > 0 else -127))
        assert rs[0] == 64 * (127 if c > 0 else -127)
    # an all-zero row gives q = 0 and s = 1
    q, s, rs = oracle.quant_act(np.zeros((3, 32), dtype=np.float32))
    assert not q.any() and np.all(s == 1.0) and not rs.any()


def test_quant_invariants():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((64, 2560)).astype(np.float32)
    X[::7] *= np.float32(1e-3)
    X[3, 5] = 40.0
    q, s, rs = oracle.quant_act(X)
    assert np.all(np.abs(q.astype(np.int32)) <= 127)          # 255 levels: -128 never occurs
    np.testing.assert_array_equal(rs, q.astype(np.int64).sum(axis=1))
    am = np.argmax(np.abs(X), axis=1)
    assert np.all(np.abs(q[np.arange(64), am].astype(np.int32)) == 127)
    # round trip: |x - q/s| <= 0.5/s (plus the rounding of x*s)
    err = np.abs(X.astype(np.float64) - q.astype(np.float64) / s[:, None].astype(np.float64))
    assert np.all(err <= (0.5 + 1e-5) / s[:, None].astype(np.float64))
    # sign symmetry (ties to even is symmetric) and power-of-two scaling
    q_neg, s_neg, _ = oracle.quant_act(-X)
    np.testing.assert_array_equal(q_neg, -q)
    assert np.array_equal(s_neg, s)
    for k in (-3, 1, 5):
        q2, s2, _ = oracle.quant_act(X * np.float32(2.0 ** k))
        np.testing.assert_array_equal(q2, q)
        np.testing.assert_array_equal(s2, s / np.float32(2.0 ** k))


def test_quant_brute_force_exact():
    """Two- and three-element rows over a grid with exact .5 ties, against
    exact rational arithmetic: s = fl32(127 / amax), q = rint(fl32(x * s))."""
    vals = [0.0, 0.5, -0.5, 1.0, -1.0, 1.5, 2.0, -2.5, 3.0, 127.0, -63.5, 0.25, 10.0, 1.27]
    vals = [float(np.float32(v)) for v in vals]
    for a in vals:
        for b in vals:
            for c in (0.0, 2.54):
                x = np.array([[a, b, c]], dtype=np.float32)
                q, s, _ = oracle.quant_act(x)
                amax = max(abs(float(v)) for v in x[0])
                if amax == 0:
                    assert s[0] == 1.0 and not q.any()
                    continue
                s_want = f32_div(127.0, amax)
                assert s[0] == s_want
                for i, v in enumerate(x[0]):
                    want = rint_half_even(Fraction(float(f32_mul(v, s_want))))
                    assert q[0, i] == max(-128, min(127, want)), (x, i)


def test_quant_bad_scale_row_is_zero():
    """A max so small that 127/max overflows gives q = 0, s = 1."""
    tiny = np.float32(1e-44)                     # subnormal: 127/tiny = inf in fp32
    q, s, _ = oracle.quant_act(np.array([[tiny, -tiny, 0.0, 0.0]], dtype=np.float32))
    assert s[0] == 1.0 and not q.any()


# ------------------------------------------------------------- RMSNorm

def test_golden_rmsnorm_examples():
    for case in _load("prelude_examples.json")["rmsnorm"]:
        x = np.array([case["x"]], dtype=np.float32)
        gain = None if case["gain"] is None else np.array(case["gain"], dtype=np.float32)
        y = oracle.rmsnorm(x, gain, case["eps"])
        np.testing.assert_array_equal(y[0], np.array(case["y"], dtype=np.float32), err_msg=case["note"])


def test_rmsnorm_constant_row_closed_form():
    """A constant row c gives g * c / sqrt(c^2 + eps), within fp32 rounding."""
    for c in (0.5, -3.0, 1e-3, 250.0):
        for eps in (0.0, 1e-5):
            y = oracle.rmsnorm(np.full((1, 96), c, dtype=np.float32), None, eps)
            want = c / math.sqrt(c * c + eps)
            np.testing.assert_allclose(y[0], want, rtol=3e-7)


def test_rmsnorm_against_fp64():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((16, 2560)).astype(np.float32)
    g = rng.uniform(0.5, 1.5, 2560).astype(np.float32)
    y = oracle.rmsnorm(X, g, 1e-5)
    X64 = X.astype(np.float64)
    want = X64 / np.sqrt(np.mean(X64 ** 2, axis=1, keepdims=True) + 1e-5) * g
    np.testing.assert_allclose(y, want, rtol=1e-6, atol=0)


def test_rmsnorm_exact_scale_invariance_with_zero_eps():
    """With eps = 0 the normalised row (and its codes) are bit-identical under
    x -> 2^k x (the sub-norm undoes a scaling of its input)."""
    rng = np.random.default_rng(6)
    X = rng.standard_normal((8, 512)).astype(np.float32)
    q0, s0, _ = oracle.quant_act(X, oracle.PRELUDE_RMSNORM, eps=0.0)
    for k in (-4, 1, 3):
        q, s, _ = oracle.quant_act(X * np.float32(2.0 ** k), oracle.PRELUDE_RMSNORM, eps=0.0)
        np.testing.assert_array_equal(q, q0)
        np.testing.assert_array_equal(s, s0)


# ------------------------------------------------------------------ FWHT

def test_golden_fwht_examples():
    cases = _load("prelude_examples.json")["fwht"]
    y = oracle.fwht(np.array([cases[0]["x"]], dtype=np.float32))
    np.testing.assert_array_equal(y[0], np.array(cases[0]["y"], dtype=np.float32))
    y = oracle.fwht(np.array([cases[1]["x"]], dtype=np.float32))
    assert np.all(y[0] == np.float32(1 / math.sqrt(8)))
    y = oracle.fwht(np.array([cases[2]["x"]], dtype=np.float32))
    np.testing.assert_allclose(y[0] * math.sqrt(2), cases[2]["y_times_sqrt2"], rtol=2e-7)


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64])
def test_fwht_equals_dense_sylvester_matrix(n):
    """Textbook routine: the dense Sylvester Hadamard matrix times x / sqrt(n)."""
    rng = np.random.default_rng(n)
    X = rng.standard_normal((5, n)).astype(np.float32)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    want = X.astype(np.float64) @ H.T / math.sqrt(n)
    got = oracle.fwht(X)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-5 * max(1.0, np.abs(want).max()))


@pytest.mark.parametrize("n", [512, 2048])
def test_fwht_invariants(n):
    rng = np.random.default_rng(n)
    X = rng.standard_normal((4, n)).astype(np.float32)
    Y = oracle.fwht(X)
    # Parseval and involution (the normalised transform is its own inverse)
    np.testing.assert_allclose(np.linalg.norm(Y, axis=1), np.linalg.norm(X, axis=1), rtol=1e-5)
    np.testing.assert_allclose(oracle.fwht(Y), X, atol=2e-5)
    e0 = np.zeros((1, n), dtype=np.float32)
    e0[0, 0] = 1
    assert np.all(oracle.fwht(e0) == np.float32(1 / math.sqrt(n)))


def test_fwht_rejects_non_power_of_two():
    with pytest.raises(oracle.OracleError):
        oracle.fwht(np.zeros((1, 12), dtype=np.float32))
    with pytest.raises(oracle.OracleError):
        oracle.quant_act(np.zeros((1, 24), dtype=np.float32), oracle.PRELUDE_FWHT)


def test_quant_with_fwht_prelude_matches_composition():
    rng = np.random.default_rng(8)
    X = rng.standard_normal((6, 512)).astype(np.float32)
    q, s, _ = oracle.quant_act(X, oracle.PRELUDE_FWHT)
    q2, s2, _ = oracle.quant_act(oracle.fwht(X))
    np.testing.assert_array_equal(q, q2)
    np.testing.assert_array_equal(s, s2)
    q, s, _ = oracle.quant_act(X, oracle.PRELUDE_RMSNORM, eps=1e-5)
    q2, s2, _ = oracle.quant_act(oracle.rmsnorm(X, None, 1e-5))
    np.testing.assert_array_equal(q, q2)
    np.testing.assert_array_equal(s, s2)
