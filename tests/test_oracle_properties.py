"""Randomised property pins for the oracle (hypothesis drives small shapes
and value grids; CPU only).

Each property follows from the definitions on the pages, not from the
oracle's own code: nnterp encyclopedia "bitnet", "The projections quantize
their inputs and weights" (per-token round(x * 127 / max|x|) to 255 levels,
weights rounded to {-1, 0, 1} * mean|W|, the output the linear map of the
rounded operands), "The two checkpoints" (four codes to a byte); the
"bitnetv2-model" README, "Special Features" (normalised Hadamard transform on
power-of-two widths).
"""
from fractions import Fraction

import numpy as np
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402
from hypothesis.extra import numpy as hnp  # noqa: E402

import oracle  # noqa: E402
from tests.exact import nearest_f32  # noqa: E402

SETTINGS = settings(max_examples=150, deadline=None)

# finite fp32 values on a wide but overflow-free range, zeros included
_f32 = st.floats(min_value=-1e6, max_value=1e6, allow_nan=False, allow_infinity=False, width=32)


def _rows(max_m=4, widths=(16, 32, 48, 64)):
    return st.sampled_from(widths).flatmap(
        lambda k: st.integers(1, max_m).flatmap(
            lambda m: hnp.arrays(np.float32, (m, k), elements=_f32)))


@SETTINGS
@given(_rows())
def test_quant_codes_follow_the_absmax_rule(X):
    """Codes lie in [-127, 127]; the largest |x| of a row maps to +-127 with
    its sign; codes are monotone in x and never flip a sign; x * s is within
    half a step (plus one fp32 rounding) of its code."""
    q, s, rs = oracle.quant_act(X)
    q = q.astype(np.int64)
    assert np.all(np.abs(q) <= 127)
    np.testing.assert_array_equal(rs, q.sum(axis=1))
    for m in range(X.shape[0]):
        x = X[m].astype(np.float64)
        amax = np.abs(x).max()
        with np.errstate(over="ignore"):
            s_ref = np.float32(127.0) / np.float32(amax) if amax > 0 else np.float32(np.inf)
        if not np.isfinite(s_ref):
            assert np.all(q[m] == 0) and s[m] == np.float32(1.0)
            continue
        j = int(np.argmax(np.abs(x)))
        assert q[m, j] == (127 if x[j] > 0 else -127)
        order = np.argsort(x, kind="stable")
        assert np.all(np.diff(q[m][order]) >= 0)
        assert np.all(q[m] * np.sign(x) >= 0)
        err = np.abs(x * float(s[m]) - q[m])
        assert np.all(err <= 0.5 + 128.0 * 2.0 ** -23)


@SETTINGS
@given(_rows(), st.integers(-20, 20))
def test_quant_codes_are_invariant_under_power_of_two_scaling(X, k):
    """Scaling a token by 2^k scales its amax by 2^k and s by 2^-k exactly, so
    the codes do not change (away from fp32 under- and overflow)."""
    amax = np.abs(X).max(axis=1)
    keep = (amax > 2.0 ** -60) & (amax < 2.0 ** 60)
    if not keep.any():
        return
    X = X[keep]
    Y = (X.astype(np.float64) * 2.0 ** k).astype(np.float32)
    if not np.all(np.isfinite(Y)) or np.any(np.abs(Y)[np.abs(X) > 0] < 2.0 ** -100):
        return
    q1, s1, _ = oracle.quant_act(X)
    q2, s2, _ = oracle.quant_act(Y)
    np.testing.assert_array_equal(q1, q2)
    np.testing.assert_array_equal(s2.astype(np.float64), s1.astype(np.float64) * 2.0 ** -k)


_w = st.floats(min_value=-4.0, max_value=4.0, allow_nan=False, allow_infinity=False, width=32)


def assert_gamma_is_rounded_mean(W, g):
    """gamma is the exact rational mean of |W| rounded to the nearest fp32
    (subnormals included, where fp32 holds fewer than 24 significant bits):
    within half an fp32 spacing at that mean, plus the few fp64 ulps the
    accumulation of the sum may add (the mean is a real number; the oracle
    sums in fp64 and rounds once)."""
    exact = sum(Fraction(float(abs(v))) for v in W.ravel()) / W.size
    near = nearest_f32(exact)
    spacing = Fraction(float(np.spacing(np.float32(min(abs(near), np.float32(3.0e38))))))
    bound = spacing / 2 + exact * Fraction(W.size + 2, 2 ** 52)
    assert abs(Fraction(float(g)) - exact) <= bound, (float(g), float(exact))


def test_gamma_of_a_single_subnormal_mean():
    """Regression case: one weight at the smallest normal fp32 (2^-126), the
    other eleven zero; the mean 2^-126 / 12 is subnormal in fp32, so gamma is
    that value rounded at the subnormal spacing 2^-149."""
    W = np.zeros((3, 4), np.float32)
    W[0, 0] = np.float32(2.0 ** -126)
    g, T, _ = oracle.quantize_weights(W)
    assert g == nearest_f32(Fraction(2) ** -126 / 12)
    assert_gamma_is_rounded_mean(W, g)
    # |W[0,0]| / gamma = 12 > 1/2: code +1; the zeros stay 0
    assert T[0, 0] == 1 and np.count_nonzero(T) == 1


@SETTINGS
@given(st.integers(1, 6).flatmap(lambda n: st.sampled_from([4, 8, 16]).flatmap(
    lambda k: hnp.arrays(np.float32, (n, k), elements=_w))))
def test_ternary_codes_follow_the_absmean_rule(W):
    """gamma is mean|W| (to fp32); t is in {-1, 0, 1}, never opposite to W,
    monotone in |W|, 0 well below gamma / 2 and +-1 well above it."""
    g, T, _ = oracle.quantize_weights(W)
    assert_gamma_is_rounded_mean(W, g)
    assert set(np.unique(T)).issubset({-1, 0, 1})
    assert np.all(T.astype(np.int64) * np.sign(W) >= 0)
    if g == 0:
        assert np.all(T == 0)
        return
    a = np.abs(W.astype(np.float64)).ravel()
    t = np.abs(T.astype(np.int64)).ravel()
    order = np.argsort(a, kind="stable")
    assert np.all(np.diff(t[order]) >= 0)
    assert np.all(t[a < 0.499 * float(g)] == 0)
    assert np.all(t[a > 0.501 * float(g)] == 1)


@SETTINGS
@given(st.integers(1, 5), st.integers(1, 6), st.sampled_from([4, 8, 12, 64]), st.data())
def test_contraction_is_the_integer_matmul(M, N, K, data):
    """acc = q . t^T exactly (int64 reference through numpy), and the packed
    round trip (four codes to a byte) returns t."""
    q = data.draw(hnp.arrays(np.int8, (M, K), elements=st.integers(-128, 127)))
    T = data.draw(hnp.arrays(np.int8, (N, K), elements=st.integers(-1, 1)))
    acc = oracle.contract(q, T)
    np.testing.assert_array_equal(acc, q.astype(np.int64) @ T.astype(np.int64).T)
    np.testing.assert_array_equal(oracle.unpack(oracle.pack(T), K), T)
    np.testing.assert_array_equal(oracle.unpack_tw2(oracle.pack_tw2(T), K), T)


@SETTINGS
@given(st.sampled_from([2, 4, 8, 16, 32]).flatmap(
    lambda n: hnp.arrays(np.float32, (2, n),
                         elements=st.floats(-100.0, 100.0, allow_nan=False, width=32))))
def test_normalised_hadamard_is_orthonormal(X):
    """The normalised transform preserves the norm and is its own inverse (to
    fp32 rounding): H / sqrt(n) is symmetric and orthogonal."""
    Y = oracle.fwht(X)
    Z = oracle.fwht(Y)
    n = X.shape[1]
    scale = np.abs(X).max() + 1e-30
    tol = 8 * n * 2.0 ** -23 * scale
    np.testing.assert_allclose(np.linalg.norm(Y.astype(np.float64), axis=1),
                               np.linalg.norm(X.astype(np.float64), axis=1), atol=tol * np.sqrt(n))
    np.testing.assert_allclose(Z, X, atol=tol)
