"""Rotary position embedding (RoPE) of key rows, for the fused RoPE + encode.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages: the Block-GTQ abstract reads the head as 2-D RoPE frequency blocks and
scores each block; the blockgtq README's quantiser takes keys after RoPE.
Quantising straight from the projection output applies RoPE inside the
encode instead.  RoPE itself is the rotary embedding of RoFormer (Su et al.,
arXiv 2104.09864): block j of a row at position p is turned by the angle
p * theta_j with theta_j = base^(-2 j / D),

    (x_a, x_b) -> (x_a cos(p theta_j) - x_b sin(p theta_j),
                   x_a sin(p theta_j) + x_b cos(p theta_j)),

with the block's two dims (a, b) = (j, j + D/2) for the half-split pairing
(rotate_half) and (2j, 2j + 1) for the interleaved one (``energy.block_dims``).
Arithmetic is float64, with no rounding of the turned values: the fused
encode quantises them as they are.
"""
import numpy as np

from .energy import block_dims


def inv_freq(head_dim, base):
    """theta_j = base^(-2 j / D) for the D/2 blocks, float64."""
    j = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * j / float(head_dim))


def apply_rope(x_rows, positions, base, pairing=0):
    """RoPE of rows x [n, D] (float64) at integer positions [n]: float64 [n, D]."""
    x = np.asarray(x_rows, dtype=np.float64)
    n, d = x.shape
    pos = np.asarray(positions, dtype=np.float64).reshape(n)
    theta = inv_freq(d, base)
    out = np.empty_like(x)
    for j, (a, b) in enumerate(block_dims(d, pairing)):
        ang = pos * theta[j]
        c, s = np.cos(ang), np.sin(ang)
        out[:, a] = x[:, a] * c - x[:, b] * s
        out[:, b] = x[:, a] * s + x[:, b] * c
    return out
