"""TurboQuant-MSE encode of one row per bit-width group (codes and norms).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages: Block-GTQ abstract / blockgtq README -- the widths chosen by the
allocator go to the TQ-MSE encoder, and the serving path keeps a packed
cache of the codes.  TQ-MSE (TurboQuant, arXiv 2504.19874, cited by the
pages): rotate, normalise, scalar-quantise each rotated coordinate with the
Lloyd-Max codebook.  Readings used here (the pages give neither):

encode, group g of width b over dims D_g (d = |D_g|):
    x_g = x[D_g]                       (fp16 input as float64)
    n   = ||x_g||                      (float64, exact input)
    y   = Pi_g x_g                     (Pi_g the fp32 table, as float64)
    u   = sqrt(d) * y / n              (u = 0 when n = 0)
    code_i = #{fp32 thresholds <= u_i} (ties go up)
    stored norm = fp16(n), round-to-nearest-even; codes use the unrounded n.

This module stops at the codes and norms.  The cache stores them in the
64-position tile format of ``tiles`` (bit-plane selector words, one region
per width group, widest group first): ``record_widths`` gives the width of
each coordinate in record order (groups width-descending, rotated-coordinate
order inside a group), the order ``tiles`` packs.  A position still costs
exactly A * D bits of codes for an average of A bits per dim (48 bytes for
D = 128 at 3 bits), plus its fp16 norms.
"""
import numpy as np

from .lloyd_max import quantise


def rotated_normalised(x_rows, dims, rotation):
    """(u [n, d], norms [n]) of one group: u = sqrt(d) Pi x / ||x|| (0 for a zero x)."""
    xg = np.asarray(x_rows, dtype=np.float64)[:, dims]
    d = len(dims)
    norms = np.sqrt(np.sum(xg * xg, axis=1))
    y = xg @ rotation.astype(np.float64).T                 # y = Pi x per row
    safe = np.where(norms > 0, norms, 1.0)
    u = np.sqrt(float(d)) * y / safe[:, None]
    u[norms == 0] = 0.0
    return u, norms


def encode_group(x_rows, dims, rotation, bits):
    """Codes [n, d] (int64) and norms [n] (float64, unrounded) of one group.

    x_rows: [n, D] float64 (exact fp16 values); rotation: fp32 [d, d].
    """
    u, norms = rotated_normalised(x_rows, dims, rotation)
    return quantise(u, bits), norms


def fp16_round(values):
    """Round float64 values to fp16 (numpy rounds to nearest even)."""
    return np.asarray(values, dtype=np.float64).astype(np.float16)


def record_widths(groups):
    """Per-position widths of a record, in record order."""
    return np.concatenate([np.full(len(dims), b, dtype=np.int64) for b, dims in groups])
