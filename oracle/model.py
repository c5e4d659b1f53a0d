"""Cache-level oracle calls: allocate, encode rows, rotate the query, decode.

TEST INFRASTRUCTURE ONLY (see the package docstring).

These mirror the library's three calls (allocate, encode-append, decode
attention) on plain arrays for one layer at a time.  The per-(layer, KV head)
tables are the group layout from the allocation, one fp32 Haar rotation per
K width group and one for V, and the fp32 Lloyd-Max codebooks.

Cache contents (the bytes the library writes, compared bit for bit):
  K tiles   uint8[1024 * k_avg_bits] per 64 positions -- ``tiles`` format
  K norms   fp16[4] per position -- slot i = group i in width-descending
            order; unused slots are +0
  V tiles   uint8[1024 * v_avg_bits] per 64 positions -- V is one group of
            all D dims at the uniform width v_avg_bits
  V norm    fp16 per position
"""
from dataclasses import dataclass

import numpy as np

from . import allocate as alloc
from . import energy, haar, lloyd_max, rope, tiles, tqmse
from .attention import attend, dequantise_keys, dequantise_values

KIND_K = 0
KIND_V = 1
MAX_GROUPS = 4


@dataclass
class Config:
    n_layers: int
    n_kv_heads: int
    n_q_heads: int
    head_dim: int = 128
    k_avg_bits: int = 3
    v_avg_bits: int = 3
    b_min: int = 1
    b_max: int = 4
    pairing: int = 0
    seed: int = 0

    @property
    def group_size(self):
        return self.n_q_heads // self.n_kv_heads



def allocate(cfg, calib_q, calib_k):
    """Widths int64 [L, Hkv, D/2] from calibration rows.

    calib_q fp16 [L, Nq, Hq, D], calib_k fp16 [L, Nk, Hkv, D].
    """
    out = np.zeros((cfg.n_layers, cfg.n_kv_heads, cfg.head_dim // 2), dtype=np.int64)
    for layer in range(cfg.n_layers):
        eq, ek = energy.block_energies(calib_q[layer], calib_k[layer], cfg.pairing)
        s = energy.block_scores(eq, ek)
        for h in range(cfg.n_kv_heads):
            out[layer, h] = alloc.greedy_allocate(s[h], cfg.k_avg_bits, cfg.b_min, cfg.b_max)
    return out


class Tables:
    """All tables of one configuration for a given allocation."""

    def __init__(self, cfg, block_widths, layers=None):
        self.cfg = cfg
        self.block_widths = np.asarray(block_widths, dtype=np.int64)
        self.codebooks = {}
        for b in range(1, lloyd_max.MAX_BITS + 1):
            self.codebooks[b] = lloyd_max.codebook_fp16(b)[0]
        self.groups = {}
        self.k_rot = {}
        self.v_rot = {}
        layers = range(cfg.n_layers) if layers is None else layers
        for layer in layers:
            for h in range(cfg.n_kv_heads):
                groups = alloc.group_layout(self.block_widths[layer, h], cfg.head_dim, cfg.pairing)
                self.groups[layer, h] = groups
                self.k_rot[layer, h] = {
                    b: haar.rotation_fp32(len(dims), cfg.seed, layer, h, KIND_K, b) for b, dims in groups}
                self.v_rot[layer, h] = haar.rotation_fp32(
                    cfg.head_dim, cfg.seed, layer, h, KIND_V, cfg.v_avg_bits)


def encode_rows(tables, layer, head, k_rows, v_rows):
    """Encode rows of one (layer, KV head): fp16 [n, D] each, as cache positions 0..n-1.

    Returns a dict with the cache bytes (k_tiles, k_norms, v_tiles, v_norm;
    the tiles padded with code 0 past row n) and the codes in record order.
    """
    k = np.asarray(k_rows, dtype=np.float16).astype(np.float64)
    v = np.asarray(v_rows, dtype=np.float16).astype(np.float64)
    return _encode(tables, layer, head, k, v)


def encode_rows_rope(tables, layer, head, k_rows, v_rows, positions, base):
    """The fused RoPE + encode: fp16 keys [n, D] taken before RoPE, turned by
    RoPE at their positions [n] with the given base (the configuration's
    pairing) in float64 and encoded without rounding the turned values;
    values as in encode_rows.  Same result layout as encode_rows."""
    k = np.asarray(k_rows, dtype=np.float16).astype(np.float64)
    k = rope.apply_rope(k, positions, base, tables.cfg.pairing)
    v = np.asarray(v_rows, dtype=np.float16).astype(np.float64)
    return _encode(tables, layer, head, k, v)


def _encode(tables, layer, head, k, v):
    """encode_rows on float64 rows k, v [n, D]."""
    cfg = tables.cfg
    n = k.shape[0]
    groups = tables.groups[layer, head]
    k_codes = []
    k_norms = np.zeros((n, MAX_GROUPS), dtype=np.float16)
    for gi, (b, dims) in enumerate(groups):
        codes, norms = tqmse.encode_group(k, dims, tables.k_rot[layer, head][b], b)
        k_codes.append(codes)
        k_norms[:, gi] = tqmse.fp16_round(norms)
    k_codes = np.concatenate(k_codes, axis=1) if k_codes else np.zeros((n, 0), dtype=np.int64)
    all_dims = np.arange(cfg.head_dim)
    v_codes, v_norm = tqmse.encode_group(v, all_dims, tables.v_rot[layer, head], cfg.v_avg_bits)
    return {"k_tiles": tiles.pack_k_tiles(k_codes, groups, cfg.k_avg_bits), "k_norms": k_norms,
            "v_tiles": tiles.pack_v_tiles(v_codes, cfg.v_avg_bits), "v_norm": tqmse.fp16_round(v_norm),
            "k_codes": k_codes, "v_codes": v_codes, "n": n}


def rotated_query(tables, layer, head, q):
    """q~ [G, D] float64 in record order: (1/sqrt(D)) (1/sqrt(d_g)) Pi_g q[D_g] per group."""
    cfg = tables.cfg
    q = np.asarray(q, dtype=np.float16).astype(np.float64)
    parts = []
    for b, dims in tables.groups[layer, head]:
        rot = tables.k_rot[layer, head][b].astype(np.float64)
        parts.append((q[:, dims] @ rot.T) / np.sqrt(float(len(dims))) / np.sqrt(float(cfg.head_dim)))
    return np.concatenate(parts, axis=1)


def decode(tables, layer, head, q, k_tiles, k_norms, v_tiles, v_norm, n):
    """Decode attention of the G query heads of one KV head over positions
    0..n-1 of the given tiles: out float64 [G, D]."""
    cfg = tables.cfg
    groups = tables.groups[layer, head]
    kc = tiles.unpack_k_tiles(k_tiles, groups, n) if n else np.zeros((0, 128), dtype=np.int64)
    vc = tiles.unpack_v_tiles(v_tiles, cfg.v_avg_bits, n) if n else np.zeros((0, 128), dtype=np.int64)
    k_hat = dequantise_keys(kc, np.asarray(k_norms)[:n], groups, tables.k_rot[layer, head], tables.codebooks,
                            cfg.head_dim)
    v_hat = dequantise_values(vc, np.asarray(v_norm)[:n], tables.v_rot[layer, head],
                              tables.codebooks[cfg.v_avg_bits], cfg.head_dim)
    q64 = np.asarray(q, dtype=np.float16).astype(np.float64)
    return attend(q64, k_hat, v_hat)


def decode_buffered(tables, layer, head, q, k_tiles, k_norms, v_tiles, v_norm, lo, hi, buf_k, buf_v):
    """Decode attention with an fp16 buffer (blockgtq README, AIME commands:
    the "withbuffer" setting keeps a few sink positions and a recent window
    unquantised): one softmax over the dequantised packed positions lo..hi-1
    of the given tiles and the buffered rows buf_k / buf_v (fp16 [n_buf, D],
    taken as they are).  out float64 [G, D]."""
    cfg = tables.cfg
    groups = tables.groups[layer, head]
    kc = tiles.unpack_k_tiles(k_tiles, groups, hi)[lo:hi] if hi > lo else np.zeros((0, 128), dtype=np.int64)
    vc = tiles.unpack_v_tiles(v_tiles, cfg.v_avg_bits, hi)[lo:hi] if hi > lo else np.zeros((0, 128), dtype=np.int64)
    k_hat = dequantise_keys(kc, np.asarray(k_norms)[lo:hi], groups, tables.k_rot[layer, head], tables.codebooks,
                            cfg.head_dim)
    v_hat = dequantise_values(vc, np.asarray(v_norm)[lo:hi], tables.v_rot[layer, head],
                              tables.codebooks[cfg.v_avg_bits], cfg.head_dim)
    bk = np.asarray(buf_k, dtype=np.float16).astype(np.float64).reshape(-1, cfg.head_dim)
    bv = np.asarray(buf_v, dtype=np.float16).astype(np.float64).reshape(-1, cfg.head_dim)
    q64 = np.asarray(q, dtype=np.float16).astype(np.float64)
    return attend(q64, np.concatenate([k_hat, bk]), np.concatenate([v_hat, bv]))
