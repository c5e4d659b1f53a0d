"""Pins for oracle/lloyd_max.py: textbook tables, closed forms, optimality by sampling."""
import math

import numpy as np
import pytest

from oracle import lloyd_max as lm


def _tol(text):
    """1.5 units in the last printed digit: Max's entries carry his own
    numerical error of about one unit there (his N = 2 level is 0.7980
    against the exact sqrt(2/pi) = 0.79788)."""
    dec = len(text.split(".")[1]) if "." in text else 0
    return 1.5 * 10.0 ** (-dec)


def test_matches_max_1960_table(golden):
    for row in golden("lloyd_max_gaussian.txt"):
        bits = int(row[0])
        # Max's 16-level MSE (0.009497) is 0.04 % below the exact value
        # (0.0095010, i.e. 20.22 dB); allow 0.05 % relative on this column.
        assert abs(lm.mse(bits) - float(row[1])) <= max(_tol(row[1]), 5e-4 * float(row[1]))
        pos = lm.centroids(bits)[1 << (bits - 1):]
        assert len(pos) == len(row) - 2
        for val, text in zip(pos, row[2:]):
            assert abs(val - float(text)) <= _tol(text), (bits, val, text)


def test_one_bit_closed_form():
    c = lm.centroids(1)
    assert c[1] == pytest.approx(math.sqrt(2.0 / math.pi), abs=1e-15)
    assert c[0] == -c[1]
    assert lm.mse(1) == pytest.approx(1.0 - 2.0 / math.pi, abs=1e-14)


def test_distortion_constants_match_recomputed_mse():
    assert lm.DISTORTION[0] == 1.0
    for b in range(1, 5):
        assert abs(lm.DISTORTION[b] - lm.mse(b)) < 1e-5
    gains = [lm.DISTORTION[b] - lm.DISTORTION[b + 1] for b in range(4)]
    assert all(gains[i] > gains[i + 1] > 0 for i in range(3))      # convex, decreasing


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_symmetry_and_midpoints(bits):
    c = lm.centroids(bits)
    t = lm.thresholds(bits)
    assert np.all(np.diff(c) > 0)
    assert np.array_equal(c, -c[::-1])
    assert t[len(t) // 2] == 0.0
    assert np.allclose(t, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=0)
    cf, tf = lm.codebook_fp16(bits)
    assert cf.dtype == np.float32 and tf.dtype == np.float32
    # the table is the binary16 rounding of the float64 levels (half an fp16 ulp)
    assert np.array_equal(cf, c.astype(np.float16).astype(np.float32))
    assert np.all(np.abs(cf.astype(np.float64) - c) <= np.abs(c) * 2.0 ** -11)
    # thresholds: exact midpoints of the stored levels, symmetric, middle one 0
    assert np.array_equal(tf.astype(np.float64), (cf[:-1].astype(np.float64) + cf[1:].astype(np.float64)) / 2)
    assert np.array_equal(tf, -tf[::-1]) and tf[len(tf) // 2] == 0.0


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_optimality_by_sampling(bits):
    """Centroid condition and MSE checked on 2e6 N(0,1) samples (brute force, not the iteration)."""
    rng = np.random.default_rng(100 + bits)
    x = rng.standard_normal(2_000_000)
    code = lm.quantise(x, bits)
    c = lm.centroids(bits)
    for k in range(len(c)):
        sel = x[code == k]
        se = sel.std() / math.sqrt(len(sel))
        assert abs(sel.mean() - c[k]) < 5 * se + 1e-4
    mse = np.mean((x - c[code]) ** 2)
    assert abs(mse - lm.mse(bits)) < 5 * np.std((x - c[code]) ** 2) / math.sqrt(len(x))


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_quantiser_is_nearest_centroid(bits):
    rng = np.random.default_rng(7)
    u = rng.standard_normal(100_000) * 1.5
    cf, tf = lm.codebook_fp16(bits)
    code = lm.quantise(u, bits)
    nearest = np.argmin(np.abs(u[:, None] - cf.astype(np.float64)[None, :]), axis=1)
    near_tie = np.min(np.abs(u[:, None] - tf.astype(np.float64)[None, :]), axis=1) < 1e-6
    assert np.array_equal(code[~near_tie], nearest[~near_tie])
    # ties go to the upper cell; zero maps to the first positive centroid
    assert np.array_equal(lm.quantise(tf.astype(np.float64), bits), np.arange(1, len(cf)))
    assert lm.quantise(np.array([0.0]), bits)[0] == 1 << (bits - 1)


def _stored_quantiser_mse(bits):
    """Exact E[(X - Q(X))^2] of the stored quantiser (binary16 levels, cells
    at their midpoints) for X ~ N(0, 1), cell by cell:
    int_a^b (x - c)^2 phi = P - (b phi(b) - a phi(a)) - 2 c (phi(a) - phi(b)) + c^2 P,
    with P = Phi(b) - Phi(a)."""
    def phi(x):
        return 0.0 if math.isinf(x) else math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)

    def xphi(x):
        return 0.0 if math.isinf(x) else x * phi(x)

    def Phi(x):
        if math.isinf(x):
            return 1.0 if x > 0 else 0.0
        return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))

    cf, tf = lm.codebook_fp16(bits)
    c = cf.astype(np.float64)
    t = np.concatenate(([-math.inf], tf.astype(np.float64), [math.inf]))
    total = 0.0
    for k in range(len(c)):
        a, b = t[k], t[k + 1]
        p = Phi(b) - Phi(a)
        total += p - (xphi(b) - xphi(a)) - 2.0 * c[k] * (phi(a) - phi(b)) + c[k] * c[k] * p
    return total


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_stored_table_distortion(bits):
    """The table both sides store (binary16 levels) keeps the Lloyd-Max
    distortion: its exact MSE is within 1e-5 relative of the float64 optimum
    and of the allocator's constant D(b), and never below the optimum."""
    d = _stored_quantiser_mse(bits)
    assert d >= lm.mse(bits) * (1 - 1e-12)
    assert abs(d - lm.mse(bits)) <= 1e-5 * lm.mse(bits)
    assert abs(d - lm.DISTORTION[bits]) <= 1e-5 + 5e-4 * lm.DISTORTION[bits]


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_stored_table_distortion_by_sampling(bits):
    """Brute force: 2e6 N(0,1) samples coded with the stored thresholds and
    reconstructed with the stored binary16 levels (not the float64 ones)
    reproduce the closed form above within 5 standard errors."""
    rng = np.random.default_rng(200 + bits)
    x = rng.standard_normal(2_000_000)
    cf, _ = lm.codebook_fp16(bits)
    err = (x - cf.astype(np.float64)[lm.quantise(x, bits)]) ** 2
    assert abs(err.mean() - _stored_quantiser_mse(bits)) < 5 * err.std() / math.sqrt(len(x))


def test_stored_levels_match_max_1960_table(golden):
    """Each stored binary16 level is within Max's printed precision (1.5 units
    of his last digit) plus half a binary16 ulp of his Table I entry; the
    largest gap over all 15 positive levels is 7.4e-4 (b = 2, 1.5107 vs 1.510)."""
    worst = 0.0
    for row in golden("lloyd_max_gaussian.txt"):
        bits = int(row[0])
        cf, _ = lm.codebook_fp16(bits)
        for val, text in zip(cf[1 << (bits - 1):].astype(np.float64), row[2:]):
            half_ulp = 2.0 ** (math.floor(math.log2(abs(val))) - 11)
            assert abs(val - float(text)) <= _tol(text) + half_ulp, (bits, val, text)
            worst = max(worst, abs(val - float(text)))
    assert worst < 7.5e-4
