"""The division-free ternary rule the weight packer uses, checked on the CPU
against IEEE division and rounding over many scales.

The absmean rule (nnterp encyclopedia "bitnet", "The projections quantize
their inputs and weights": weights rounded to {-1, 0, 1} * mean|W|) gives
t = clamp(rint(fl(w / gamma)), -1, 1).  The packer never divides: it marks
t != 0 exactly when |w| > RD_f32(gamma * (1/2 + 2^-25)), where the product is
exact in fp64 and RD rounds down to fp32.  The argument: rint(fl(q)) != 0
exactly when fl(q) > 1/2; the fp32 numbers next to 1/2 are 1/2 and
1/2 + 2^-24, so fl(q) > 1/2 exactly when q > 1/2 + 2^-25 (the tie rounds to
the even 1/2); for an fp32 |w| the strict compare against the exact product
and against its round-down agree.  This file restates that rule in numpy and
compares it with numpy's IEEE float32 division and rint for thousands of
gamma mantissas across the exponent range, subnormal gamma included, at the
weights that straddle each threshold.  No GPU and no oracle are involved:
it checks the claim the kernel is built on.
"""
import numpy as np


def _rd_f32(x64):
    """Round fp64 values down to fp32."""
    f = x64.astype(np.float32)
    over = f.astype(np.float64) > x64
    f[over] = np.nextafter(f[over], np.float32(-np.inf))
    return f


def _threshold(g32):
    return _rd_f32(g32.astype(np.float64) * (0.5 + 2.0 ** -25))


def _by_division(w32, g32):
    with np.errstate(over="ignore", under="ignore", divide="ignore", invalid="ignore"):
        q = np.float32(w32) / np.float32(g32)
        t = np.clip(np.rint(q), -1, 1)
    return np.where(g32 == 0, 0, t).astype(np.int8)


def _by_threshold(w32, g32):
    thr = _threshold(g32)
    t = np.where(np.abs(w32) > thr, np.sign(w32), 0)
    return np.where(g32 == 0, 0, t).astype(np.int8)


def _gammas(rng, count):
    """Random fp32 mantissas at every exponent from the subnormals up to
    2^100, plus hand-picked edges."""
    exps = rng.integers(-149, 100, size=count)
    mant = rng.integers(0, 1 << 23, size=count)
    normal = (np.float64(1.0) + mant / float(1 << 23)) * np.exp2(exps.astype(np.float64))
    sub = mant.astype(np.float64) * 2.0 ** -149                      # subnormal gammas
    g = np.where(exps < -126, sub, normal).astype(np.float32)
    edges = np.array([2.0 ** -149, 3 * 2.0 ** -149, 2.0 ** -127, 2.0 ** -126,
                      1.1754942e-38, 0.5, 1.0, 1.5, 0.015957, 3.0e38], np.float32)
    g = np.concatenate([g, edges])
    return g[g > 0]


def test_threshold_rule_equals_division_near_every_boundary():
    rng = np.random.default_rng(2024)
    g = _gammas(rng, 20000)
    thr = _threshold(g)
    # the fp32 weights on both sides of the threshold, and of the exact
    # boundary gamma / 2 and gamma * 1.5 (the clamp)
    cands = [thr, np.nextafter(thr, np.float32(np.inf)), np.nextafter(thr, np.float32(-np.inf)),
             (g.astype(np.float64) * 0.5).astype(np.float32), g, g * np.float32(1.5),
             np.nextafter(g * np.float32(0.5), np.float32(np.inf))]
    for w in cands:
        for sign in (1, -1):
            ws = (sign * w).astype(np.float32)
            np.testing.assert_array_equal(_by_threshold(ws, g), _by_division(ws, g))


def test_threshold_rule_equals_division_on_random_weights():
    rng = np.random.default_rng(7)
    g = _gammas(rng, 2000)
    for _ in range(20):
        scale = np.exp2(rng.uniform(-3, 3, size=g.size)).astype(np.float32)
        with np.errstate(over="ignore"):
            w = (g * scale * rng.choice([-1, 1], size=g.size)).astype(np.float32)
        ok = np.isfinite(w)                    # inputs must be finite
        np.testing.assert_array_equal(_by_threshold(w[ok], g[ok]), _by_division(w[ok], g[ok]))


def test_zero_gamma_and_zero_weights():
    g = np.array([0.0, 0.0, 1e-3, 2.0 ** -149], np.float32)
    w = np.array([5.0, 0.0, 0.0, -0.0], np.float32)
    np.testing.assert_array_equal(_by_threshold(w, g), np.zeros(4, np.int8))
    np.testing.assert_array_equal(_by_division(w, g), np.zeros(4, np.int8))
