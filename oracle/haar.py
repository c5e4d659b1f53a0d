"""Seeded Haar-random rotations (the TQ-MSE random rotation).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages: TurboQuant-MSE, which Block-GTQ builds on (Block-GTQ abstract; blockgtq
README, method blurb), quantises a vector after a random rotation; the pages
do not say how the rotation is drawn or grouped.  Reading used here: one Haar
orthogonal matrix per (layer, KV head, K or V, bit-width group), drawn as

  SplitMix64 stream  (Steele, Lea, Flood 2014, "Fast splittable PRNGs")
  -> Box-Muller normals (Box & Muller 1958)
  -> QR of the d x d Gaussian matrix, Q := Q diag(sign(diag R))
     (Mezzadri 2007, "How to generate random matrices from the classical
     compact groups", which makes Q exactly Haar distributed),

in float64, then rounded once to fp32: the fp32 matrix is the table both the
encoder and the decoder use.

The stream key for a matrix hashes (seed, layer, head, kind, width) with one
SplitMix64 step per field: key <- next() of a generator started at state
(key XOR field).  kind is 0 for K and 1 for V; width is the group's bit width
(V uses its uniform width).  The d*d Gaussian entries fill the matrix in
row-major order, two per uniform pair (cos then sin).
"""
import math

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15


def _mix64(z):
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


class SplitMix64:
    """The SplitMix64 generator: state += gamma; output = mix(state)."""

    def __init__(self, state):
        self.state = state & MASK64

    def next(self):
        self.state = (self.state + GOLDEN_GAMMA) & MASK64
        return _mix64(self.state)

    def uniform(self):
        """Uniform on [0, 1) with 53 random bits."""
        return (self.next() >> 11) * (1.0 / (1 << 53))


def rotation_key(seed, layer, head, kind, width):
    key = seed & MASK64
    for field in (layer, head, kind, width):
        key = SplitMix64(key ^ (field & MASK64)).next()
    return key


def gaussian_matrix(d, key):
    """d x d standard normal entries from the stream ``key`` (row-major)."""
    gen = SplitMix64(key)
    n = d * d
    out = []
    while len(out) < n:
        u1 = 1.0 - gen.uniform()          # (0, 1]
        u2 = gen.uniform()                # [0, 1)
        r = math.sqrt(-2.0 * math.log(u1))
        out.append(r * math.cos(2.0 * math.pi * u2))
        out.append(r * math.sin(2.0 * math.pi * u2))
    return np.array(out[:n], dtype=np.float64).reshape(d, d)


def haar_rotation(d, key):
    """Haar-distributed d x d orthogonal matrix in float64."""
    g = gaussian_matrix(d, key)
    q, r = np.linalg.qr(g)
    s = np.sign(np.diag(r))
    s[s == 0] = 1.0
    return q * s[np.newaxis, :]


def rotation_fp32(d, seed, layer, head, kind, width):
    """The stored table: the float64 Haar matrix rounded once to fp32."""
    return haar_rotation(d, rotation_key(seed, layer, head, kind, width)).astype(np.float32)
