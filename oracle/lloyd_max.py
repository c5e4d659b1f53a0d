"""Gaussian Lloyd-Max scalar quantiser (the TQ-MSE codebook).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages: the Block-GTQ abstract ("built on TurboQuant-MSE (TQ-MSE)") and the
blockgtq README (TQ-MSE encoder); TurboQuant (arXiv 2504.19874) is the cited
source of TQ-MSE: after a random rotation each coordinate of a normalised
vector is quantised with the optimal (Lloyd-Max) scalar quantiser of its
distribution.  The pages do not print the codebook; the reading used here is
the N(0, 1) Lloyd-Max quantiser applied to u = sqrt(d) * y / ||x|| (see
``tqmse``).  Pinned against Max (1960), "Quantizing for minimum distortion",
Table I, in ``tests/test_oracle_lloyd_max.py``.

Algorithm (Lloyd 1957/1982, Max 1960): alternate the two optimality
conditions until nothing changes --
  * each threshold is the midpoint of its two neighbouring centroids;
  * each centroid is the conditional mean of X ~ N(0,1) on its cell,
    E[X | a < X < b] = (phi(a) - phi(b)) / (Phi(b) - Phi(a)).
The codebook is symmetric, so only the positive half is iterated and the
negative half is its mirror image (which makes the middle threshold 0
exactly).
"""
import functools
import math

import numpy as np

# Distortion constants the greedy allocator uses for the marginal gain of one
# more bit.  They are the N(0,1) Lloyd-Max mean-squared errors to six digits
# (Max 1960); both the oracle and the library use these literal values, and
# ``tests/test_oracle_lloyd_max.py`` checks them against ``mse()`` below.
DISTORTION = {0: 1.0, 1: 0.363380, 2: 0.117482, 3: 0.034548, 4: 0.009497}

MAX_BITS = 4


def _phi(x):
    if math.isinf(x):
        return 0.0
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _Phi(x):
    if x == math.inf:
        return 1.0
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def _cond_mean(a, b):
    """E[X | a < X < b] for X ~ N(0, 1)."""
    return (_phi(a) - _phi(b)) / (_Phi(b) - _Phi(a))


@functools.lru_cache(maxsize=None)
def positive_centroids(bits, tol=1e-15, max_iter=100000):
    """Positive half of the 2**bits-level Lloyd-Max codebook, ascending, float64.

    Starts from evenly spaced points on (0, 4) and alternates the two
    optimality conditions until no centroid moves by more than ``tol``
    (the iteration settles into last-ulp oscillation, never an exact fixed
    point, for 8 and 16 levels).
    """
    if bits < 1 or bits > MAX_BITS:
        raise ValueError("bits must be in 1..4")
    half = 1 << (bits - 1)
    if half == 1:
        return (_cond_mean(0.0, math.inf),)         # sqrt(2/pi)
    c = [(k + 0.5) * 4.0 / half for k in range(half)]
    for _ in range(max_iter):
        t = [0.0] + [0.5 * (c[k] + c[k + 1]) for k in range(half - 1)] + [math.inf]
        new = [_cond_mean(t[k], t[k + 1]) for k in range(half)]
        moved = max(abs(a - b) for a, b in zip(new, c))
        c = new
        if moved <= tol:
            break
    return tuple(c)


def centroids(bits):
    """All 2**bits centroids, ascending, float64 (exactly antisymmetric)."""
    pos = positive_centroids(bits)
    return np.array([-v for v in reversed(pos)] + list(pos), dtype=np.float64)


def thresholds(bits):
    """The 2**bits - 1 cell boundaries (midpoints), ascending, float64."""
    c = centroids(bits)
    return 0.5 * (c[:-1] + c[1:])


def mse(bits):
    """Mean-squared error of the quantiser on N(0, 1), float64.

    With the centroid condition met, E[(X - Q(X))^2] = 1 - sum_k P_k c_k^2.
    """
    c = centroids(bits)
    t = np.concatenate(([-math.inf], thresholds(bits), [math.inf]))
    total = 0.0
    for k in range(len(c)):
        p = _Phi(t[k + 1]) - _Phi(t[k])
        total += p * c[k] * c[k]
    return 1.0 - total


def codebook_fp16(bits):
    """The stored tables: centroids rounded once to binary16 (kept as exact
    float32 values) and the cell boundaries at the exact midpoints of those
    rounded centroids.

    Reading: the pages leave the codebook's storage precision open; the
    decode multiplies codes' centroids with fp16 operands, so the table is
    the binary16 rounding of the float64 Lloyd-Max levels (a relative shift of
    at most 2**-12 per level).  Thresholds are the nearest-neighbour cell
    boundaries of that table: (C[k] + C[k+1]) / 2, exact in float32.
    """
    c16 = centroids(bits).astype(np.float16).astype(np.float32)
    th = ((c16[:-1].astype(np.float64) + c16[1:].astype(np.float64)) / 2.0).astype(np.float32)
    assert np.array_equal(th.astype(np.float64), (c16[:-1].astype(np.float64) + c16[1:].astype(np.float64)) / 2.0)
    return c16, th


def quantise(u, bits):
    """Code of each element of ``u``: the number of thresholds <= u.

    A value equal to a threshold goes to the upper cell; u = 0 gives code
    2**(bits-1), the first positive centroid.  ``u`` may be float64 (the
    oracle) -- the thresholds are compared as their exact fp32 values.
    """
    _, th = codebook_fp16(bits)
    return np.searchsorted(th.astype(np.float64), np.asarray(u, dtype=np.float64), side="right").astype(np.int64)
