"""Label-free per-RoPE-block Q/K energy score.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages: the Block-GTQ abstract (a label-free energy score for every RoPE
block, computed separately per layer and KV head) and the blockgtq README
(the score combines Q and K, taken from saved calibration activations).  The
formula is not printed.  Reading used here:

  under RoPE, q . k = sum_j q_j^T R(theta_j (m - n)) k_j over the D/2
  two-dimensional blocks j; averaged over the relative phase,
  E[(q_j^T R k_j)^2] = ||q_j||^2 ||k_j||^2 / 2, so the score of block j is

      s_j = EQ_j * EK_j,
      EQ_j = sum over calibration rows and the G query heads of the KV group
             of ||q_{h,j}||^2,
      EK_j = sum over calibration rows of ||k_j||^2

  (the constant 1/2 and the row counts do not change the argmax, so they
  are left out).  Block j holds dims (j, j + D/2) for the half-split RoPE
  pairing and (2j, 2j + 1) for the interleaved pairing.

The sums are exact: an fp16 value times 2**24 is an integer below 2**40, so
EQ and EK are integers in units of 2**-48.  The score is the float64 product
float(EQ) * float(EK) of the two correctly rounded conversions.
"""
import numpy as np

FIXED_POINT_SHIFT = 24          # fp16 * 2**24 is an exact integer


def block_dims(head_dim, pairing):
    """List of (dim_a, dim_b) for the head_dim/2 RoPE blocks."""
    half = head_dim // 2
    if pairing == 0:
        return [(j, j + half) for j in range(half)]
    if pairing == 1:
        return [(2 * j, 2 * j + 1) for j in range(half)]
    raise ValueError("pairing must be 0 (half-split) or 1 (interleaved)")


def fp16_to_fixed(x):
    """Exact integers x * 2**24 of an fp16 array (as int64)."""
    x = np.asarray(x, dtype=np.float16).astype(np.float64) * float(1 << FIXED_POINT_SHIFT)
    xi = x.astype(np.int64)
    assert np.array_equal(xi.astype(np.float64), x)
    return xi


def sum_of_squares_exact(xi):
    """Exact sum of squares of an int64 array (|x| < 2**40) as a Python int.

    x = hi * 2**20 + lo with 0 <= lo < 2**20, so
    x^2 = hi^2 * 2**40 + 2 hi lo * 2**20 + lo^2 and each partial sum fits
    in int64 for fewer than 2**23 terms.
    """
    xi = np.asarray(xi, dtype=np.int64).ravel()
    if xi.size >= (1 << 23):
        raise ValueError("too many terms for the exact int64 split")
    hi = xi >> 20
    lo = xi - (hi << 20)
    s_hh = int(np.sum(hi * hi))
    s_hl = int(np.sum(hi * lo))
    s_ll = int(np.sum(lo * lo))
    return (s_hh << 40) + (s_hl << 21) + s_ll


def block_energies(calib_q, calib_k, pairing=0):
    """Exact EQ, EK for one layer.

    calib_q: fp16 [Nq, Hq, D]; calib_k: fp16 [Nk, Hkv, D].  Query head h
    belongs to KV head h // G with G = Hq / Hkv.  Returns two nested lists of
    Python ints, [Hkv][D/2] each, in units of 2**-48.
    """
    calib_q = np.asarray(calib_q, dtype=np.float16)
    calib_k = np.asarray(calib_k, dtype=np.float16)
    _, hq, d = calib_q.shape
    _, hkv, d2 = calib_k.shape
    assert d == d2 and hq % hkv == 0
    g = hq // hkv
    qi = fp16_to_fixed(calib_q)
    ki = fp16_to_fixed(calib_k)
    eq = [[0] * (d // 2) for _ in range(hkv)]
    ek = [[0] * (d // 2) for _ in range(hkv)]
    for kvh in range(hkv):
        for j, (a, b) in enumerate(block_dims(d, pairing)):
            qsel = qi[:, kvh * g:(kvh + 1) * g, :][:, :, [a, b]]
            eq[kvh][j] = sum_of_squares_exact(qsel)
            ek[kvh][j] = sum_of_squares_exact(ki[:, kvh, [a, b]])
    return eq, ek


def block_scores(eq, ek):
    """s_j = float(EQ_j) * float(EK_j), float64 [Hkv][D/2]."""
    return np.array([[float(a) * float(b) for a, b in zip(rq, rk)] for rq, rk in zip(eq, ek)],
                    dtype=np.float64)
