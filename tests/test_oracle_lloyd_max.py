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
