"""Pins for the oracle's weight side: absmean scale, ternary codes, packing.

Sources: nnterp encyclopedia "bitnet", "The projections quantize their inputs
and weights" (weights rounded to {-1, 0, 1} * mean|W|, stored ternary four to
a byte with a weight_scale; a 0.1 * mean|W| edit to one weight is re-ternarised
away); "BitNet b1.58 2B4T", "Model Details" (absmean quantisation).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests.exact import f32_div, nearest_f32, rint_half_even

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_golden_ternary_examples():
    for case in _load("ternary_examples.json")["cases"]:
        W = np.array(case["W"], dtype=np.float32)
        g = oracle.absmean(W)
        assert g == np.float32(case["gamma"]), case["note"]
        t = oracle.ternarize(W, g)
        np.testing.assert_array_equal(t, np.array(case["t"], dtype=np.int8), err_msg=case["note"])


def test_equal_magnitude_gives_sign():
    """Closed form: every |W| = c gives gamma = c and t = sign(W) exactly."""
    rng = np.random.default_rng(11)
    for c in (0.02, 1.0, 3.0e-5, 0.7):
        W = np.where(rng.random((37, 96)) < 0.5, -1.0, 1.0).astype(np.float32) * np.float32(c)
        g = oracle.absmean(W)
        assert g == np.float32(c)
        np.testing.assert_array_equal(oracle.ternarize(W, g), np.sign(W).astype(np.int8))


def test_gamma_matches_exact_mean():
    """gamma is the exact mean of |W| rounded once to fp32 (fsum is exact here)."""
    rng = np.random.default_rng(3)
    for shape in [(1, 1), (7, 13), (64, 256), (300, 517)]:
        W = (rng.standard_normal(shape) * 0.02).astype(np.float32)
        exact = sum(Fraction(float(abs(v))) for v in W.ravel()) / W.size
        got = oracle.absmean(W)
        want = nearest_f32(exact)
        # fp64 accumulation can differ from the exact sum only in the last
        # fp64 bits; that moves the fp32 result only next to a midpoint.
        if got != want:
            ulp = np.spacing(want)
            assert abs(Fraction(float(got)) - exact) <= Fraction(float(ulp)) * Fraction(1, 2) * (1 + Fraction(1, 10**6))


def test_ternary_invariants():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((128, 512)) * 0.02).astype(np.float32)
    g = oracle.absmean(W)
    t = oracle.ternarize(W, g)
    assert set(np.unique(t)).issubset({-1, 0, 1})
    big = np.abs(W) >= 1.5 * g
    small = np.abs(W) < 0.5 * g
    np.testing.assert_array_equal(t[big], np.sign(W[big]).astype(np.int8))
    assert np.all(t[small] == 0)
    # between the thresholds the code is the sign or 0, never the opposite sign
    mid = ~big & ~small
    assert np.all((t[mid] == 0) | (t[mid] == np.sign(W[mid])))


def test_ternary_brute_force_exact():
    """Every code equals rint(fl32(W / gamma)) computed with exact rationals,
    over random tiny matrices drawn from a grid that hits the .5 ties."""
    rng = np.random.default_rng(7)
    grid = np.array([-2.5, -2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2, 2.5, 0.25, -0.75],
                    dtype=np.float32)
    for _ in range(400):
        W = rng.choice(grid, size=(2, 4)).astype(np.float32)
        g = oracle.absmean(W)
        exact_g = nearest_f32(sum(Fraction(float(abs(v))) for v in W.ravel()) / 8)
        assert g == exact_g
        t = oracle.ternarize(W, g)
        for idx, w in np.ndenumerate(W):
            if exact_g == 0:
                want = 0
            else:
                r = f32_div(w, exact_g)
                want = max(-1, min(1, rint_half_even(Fraction(float(r)))))
            assert t[idx] == want, (W, g, idx)


def test_zero_fraction_matches_gaussian_closed_form():
    """For W ~ N(0, s^2), gamma -> s*sqrt(2/pi) and P(t = 0) -> erf(1/sqrt(4*pi))
    = 0.3101 (the "about one third zeros" of the prefill workload)."""
    rng = np.random.default_rng(0)
    W = (rng.standard_normal((6912, 2560), dtype=np.float32) * np.float32(0.02))
    g = oracle.absmean(W)
    assert abs(float(g) / (0.02 * math.sqrt(2 / math.pi)) - 1) < 1e-3
    t = oracle.ternarize(W, g)
    frac0 = float(np.mean(t == 0))
    assert abs(frac0 - math.erf(1 / math.sqrt(4 * math.pi))) < 0.002
    assert abs(math.erf(1 / math.sqrt(4 * math.pi)) - 0.3101) < 1e-4


def test_reternarize_is_idempotent():
    """Re-ternarising gamma * t returns t, with gamma' = gamma * (nonzero fraction)."""
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((33, 64)) * 0.02).astype(np.float32)
    g = oracle.absmean(W)
    t = oracle.ternarize(W, g)
    W2 = (t.astype(np.float32) * g).astype(np.float32)
    g2 = oracle.absmean(W2)
    nnz = int(np.count_nonzero(t))
    assert g2 == nearest_f32(Fraction(float(g)) * nnz / W.size)
    np.testing.assert_array_equal(oracle.ternarize(W2, g2), t)


def test_single_weight_edit_is_absorbed():
    """Adding 0.1 * mean|W| to one weight changes at most that weight's code
    (nnterp "bitnet": such an edit is re-ternarised away)."""
    rng = np.random.default_rng(21)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    g = oracle.absmean(W)
    t = oracle.ternarize(W, g)
    for i in rng.integers(0, W.size, size=20):
        W2 = W.copy().ravel()
        W2[i] = W2[i] + np.float32(0.1) * g
        W2 = W2.reshape(W.shape)
        t2 = oracle.ternarize(W2, oracle.absmean(W2))
        diff = np.flatnonzero((t2 != t).ravel())
        assert diff.size == 0 or (diff.size == 1 and diff[0] == i)


def test_golden_pack_example():
    ex = _load("pack_example.json")
    t = np.array([ex["t"]], dtype=np.int8)
    p = oracle.pack(t)
    assert p.shape == (1, 16)
    np.testing.assert_array_equal(p[0], np.array(ex["packed"], dtype=np.uint8))


def test_golden_tw2_example():
    ex = _load("tw2_example.json")
    t = np.array([ex["t"]], dtype=np.int8)
    p = oracle.pack_tw2(t)
    assert p.shape == (1, 4)
    np.testing.assert_array_equal(p[0], np.array(ex["tw2"], dtype=np.uint8))
    np.testing.assert_array_equal(oracle.unpack_tw2(p, 16), t)


@pytest.mark.parametrize("K", [16, 64, 2560, 6912])
def test_tw2_roundtrip_and_bit_positions(K):
    """Both layouts hold the same codes: each unpacks to t, a direct bit read
    of TW2 gives t + 1, and code 3 never appears."""
    rng = np.random.default_rng(K + 7)
    N = 3
    t = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    p = oracle.pack_tw2(t)
    assert p.shape == (N, K // 4)
    np.testing.assert_array_equal(oracle.unpack_tw2(p, K), t)
    np.testing.assert_array_equal(oracle.unpack(oracle.pack(t), K), t)
    for n in range(N):
        for k in list(range(min(K, 24))) + [K - 1]:
            assert ((p[n, k // 4] >> (2 * (k % 4))) & 3) == t[n, k] + 1
    codes = np.stack([(p >> s) & 3 for s in (0, 2, 4, 6)], axis=-1)
    assert not np.any(codes == 3)
    bad = p.copy()
    bad[0, 0] |= 3
    with pytest.raises(oracle.OracleError):
        oracle.unpack_tw2(bad, K)


@pytest.mark.parametrize("K", [16, 48, 64, 80, 256, 2560, 6912])
def test_pack_roundtrip_and_padding(K):
    rng = np.random.default_rng(K)
    N = 5
    t = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    p = oracle.pack(t)
    ldw = 16 * ((K + 63) // 64)
    assert p.shape == (N, ldw)
    np.testing.assert_array_equal(oracle.unpack(p, K), t)
    # code 3 never appears; padded positions hold code 1
    codes = np.stack([(p >> s) & 3 for s in (0, 2, 4, 6)], axis=-1)
    assert not np.any(codes == 3)
    # each code pair decodes independently: check with a direct bit read
    for n in range(N):
        for k in list(range(min(K, 40))) + [K - 1]:
            byte = p[n, 4 * (k // 16) + (k % 4)]
            assert ((byte >> (2 * ((k % 16) // 4))) & 3) == t[n, k] + 1
        for k in range(K, 4 * ldw):
            byte = p[n, 4 * (k // 16) + (k % 4)]
            assert ((byte >> (2 * ((k % 16) // 4))) & 3) == 1


def test_packed_bytes_per_weight():
    """Four codes to a byte: a 2560 x 6912 weight packs into N*K/4 bytes."""
    assert oracle.packed_row_bytes(2560) * 6912 == 6912 * 2560 // 4
    assert oracle.packed_row_bytes(6912) * 2560 == 4423680
