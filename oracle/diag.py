"""Per-layer logit MAE of a packed key cache.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Pages: the Block-GTQ abstract (Block-GTQ keeps the RoPE query-key logits
closer to exact: a lower per-layer MAE than uniform TQ-MSE at 2 and 3 bits
per dim, with only K quantised) and the blockgtq README, bit allocation
(`bench_perlayer_diag.py ... --avg-bits 3 --window-M 1024`, per-layer kernel
MAE table).  The pages do not define the window or the averaging; the
reading used here is the plain one:

* the window is M consecutive cached positions w0 .. w0+M-1, with the
  queries at the same positions;
* every causal pair (query i, key j), 0 <= j <= i < M, counts once;
* the logit is q . k / sqrt(D) (the softmax logit of decode attention), so
  for query head h of the KV group

      MAE_h = mean_{0 <= j <= i < M} | q_{i,h} . (k_j - k_hat_j) | / sqrt(D)

  with k the exact fp16 keys and k_hat their dequantised copies (the same
  dequantisation as decode attention, ``attention.dequantise_keys``).

Only keys are quantised here (the pages' "K-only" diagnostic).  A layer's
MAE is the mean over its query heads (every head has the same pair count).
Arithmetic is float64.
"""
import numpy as np

from . import tiles
from .attention import dequantise_keys


def causal_pair_count(m):
    """Number of pairs (i, j) with 0 <= j <= i < m."""
    return m * (m + 1) // 2


def logit_errors(q, k, k_hat):
    """Per-pair logit errors [G, M, M] (query i, key j), zero above the diagonal.

    q float [M, G, D] queries at the window's positions, k / k_hat float
    [M, D] exact and dequantised keys at the same positions.
    """
    q = np.asarray(q, dtype=np.float64)
    err = np.asarray(k, dtype=np.float64) - np.asarray(k_hat, dtype=np.float64)    # [M, D]
    d = q.shape[-1]
    delta = np.einsum("igd,jd->gij", q, err) / np.sqrt(float(d))
    m = q.shape[0]
    causal = np.tril(np.ones((m, m), dtype=bool))
    return np.where(causal[None], delta, 0.0)


def logit_mae(tables, layer, head, q_rows, k_rows, k_tiles, k_norms, w0=0):
    """MAE_h for the G query heads of one (layer, KV head): float64 [G].

    q_rows fp16 [M, G, D]: the queries at positions w0 .. w0+M-1.
    k_rows fp16 [M, D]: the exact keys cached at those positions.
    k_tiles / k_norms: the packed cache of positions 0 .. w0+M-1 (the
    ``model.encode_rows`` format, or the library's bytes).
    """
    q = np.asarray(q_rows, dtype=np.float16).astype(np.float64)
    k = np.asarray(k_rows, dtype=np.float16).astype(np.float64)
    m = q.shape[0]
    if m == 0:
        return np.zeros(q.shape[1], dtype=np.float64)
    groups = tables.groups[layer, head]
    codes = tiles.unpack_k_tiles(k_tiles, groups, w0 + m)[w0:w0 + m]
    k_hat = dequantise_keys(codes, np.asarray(k_norms)[w0:w0 + m], groups, tables.k_rot[layer, head],
                            tables.codebooks, tables.cfg.head_dim)
    delta = logit_errors(q, k, k_hat)
    return np.abs(delta).sum(axis=(1, 2)) / causal_pair_count(m)
