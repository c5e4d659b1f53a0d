"""Pins for oracle/haar.py: published SplitMix64 outputs, orthogonality, Haar statistics."""
import math

import numpy as np
import pytest
from scipy import stats

from oracle import haar


def test_splitmix64_reference_outputs(golden):
    for row in golden("splitmix64.txt"):
        g = haar.SplitMix64(int(row[0]))
        assert [g.next() for _ in row[1:]] == [int(h, 16) for h in row[1:]]


def test_box_muller_normals_are_standard_normal():
    z = haar.gaussian_matrix(200, haar.rotation_key(3, 1, 2, 0, 3)).ravel()   # 40000 samples
    assert abs(z.mean()) < 4 / math.sqrt(z.size)
    assert abs(z.var() - 1) < 4 * math.sqrt(2 / z.size)
    assert stats.kstest(z, "norm").pvalue > 1e-4


@pytest.mark.parametrize("d", [2, 8, 56, 128])
def test_orthogonal_and_preserves_dot_products(d):
    q = haar.haar_rotation(d, haar.rotation_key(11, 0, 1, 0, 2))
    assert np.abs(q.T @ q - np.eye(d)).max() < 1e-12
    rng = np.random.default_rng(d)
    a, b = rng.standard_normal(d), rng.standard_normal(d)
    assert (q @ a) @ (q @ b) == pytest.approx(a @ b, rel=1e-12, abs=1e-12)


def test_keys_are_distinct_per_field_and_deterministic():
    keys = {haar.rotation_key(5, l, h, k, w) for l in range(3) for h in range(3) for k in range(2) for w in range(5)}
    assert len(keys) == 3 * 3 * 2 * 5
    a = haar.rotation_fp32(16, 5, 1, 1, 0, 3)
    b = haar.rotation_fp32(16, 5, 1, 1, 0, 3)
    assert np.array_equal(a, b) and a.dtype == np.float32


def test_haar_statistics():
    """Columns of a Haar matrix are uniform on the sphere: E[Q_ij^2] = 1/d; the
    2x2 rotation angle is uniform (the sign fix of Mezzadri 2007 is what makes it so)."""
    d = 4
    sq = np.zeros((d, d))
    angles = []
    n = 1500
    for i in range(n):
        q = haar.haar_rotation(d, haar.rotation_key(i, 0, 0, 0, 1))
        sq += q * q
        q2 = haar.haar_rotation(2, haar.rotation_key(i, 9, 0, 0, 1))
        angles.append(math.atan2(q2[1, 0], q2[0, 0]))
    sq /= n
    assert np.abs(sq - 1.0 / d).max() < 0.03
    assert stats.kstest((np.array(angles) + math.pi) / (2 * math.pi), "uniform").pvalue > 1e-4
