"""The packed-cache tile format: where every code bit of a 64-token tile goes.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages only say that the serving path decodes attention from a packed
cache (Block-GTQ abstract, its serving path; blockgtq README);
they give no format.  This module defines the one the library stores, bit by
bit, so that both sides pack identically.  Codes are those of ``tqmse``
(record order: width groups widest first, rotated coordinates in order).

Terms
  tile       64 consecutive cache positions of one (layer, sequence, KV head)
  lane       L = 4 g + t, g = L // 4 in 0..7, t = L % 4 in 0..3
  selector   a 32-bit word of 8 nibbles; nibble n holds one code at bits
             [4n, 4n + 4) (its unused high bits are 0)

K, per width group (width b, size d, group coordinates i = 0..d-1):
  chunk j holds coordinates 16j .. 16j+15; it is full when 16j + 16 <= d,
  otherwise it is the group's partial chunk with r = d - 16j coordinates.
  Selector (chunk j, M-tile mu in 0..3, lane L), nibble n:
      token      = 16 mu + g + 8 * (n >= 4)
      coordinate = 16 j + 4 t + (n % 4)
V (width vb, coordinates 0..127):
  selector (dim-tile m in 0..7, token step kappa in 0..3, lane L), nibble n:
      coordinate = 16 m + g + 8 * (n >= 4)
      token      = 16 kappa + (2t, 2t+1, 2t+8, 2t+9)[n % 4]

Quartet: four selectors s0..s3 of one lane at width b stored as b plane words
(M1 = 0x11111111, M3 = 0x33333333, M4 = 0x44444444):
  b = 1: P = (s0&M1) | (s1&M1)<<1 | (s2&M1)<<2 | (s3&M1)<<3
  b = 2: A = (s0&M3) | (s1&M3)<<2,  B = (s2&M3) | (s3&M3)<<2
  b = 3: A, B as for b = 2, and H = (s0&M4)>>2 | (s1&M4)>>1 | (s2&M4) | (s3&M4)<<1
  b = 4: s0, s1, s2, s3
Stored symbol: widths 1..3 store the code c itself.  Width 4 stores it in
sign-magnitude form,
  sigma(c) = c - 8           for c >= 8   (the 8 positive levels, 0..7)
  sigma(c) = 8 + (7 - c)     for c < 8    (their negatives, 8..15),
so bit 3 of a symbol is the sign of its level and bits 0..2 index |level|
among the positive levels: the Lloyd-Max codebook is symmetric
(C[15 - c] = -C[c]), so symbol s stands for (-1)^[s >= 8] C[8 + s % 8].  The
selectors below hold symbols; pack / unpack convert.

A quartet region is b words x 32 lanes, word-major (word k of lane L at
index 32 k + L).  K quartets: one per full chunk, s_mu for mu = 0..3.  V
quartets: one per dim-tile m, s_kappa for kappa = 0..3.

K tile (1024 * k_avg_bits bytes): group regions widest group first; in each,
the full chunks' quartets in chunk order (b x 32 words each), then the
partial chunk (r = d - 16j coordinates, r even):
  * lanes with a full quad (t < nf = r // 4) store their quartet as above,
    word k of lane (g, t) at index 8 nf k + (g nf + t);
  * if r % 4 == 2, the eight lanes with t = nf hold two real members per
    token (nibbles 0, 1, 4, 5).  Their half selectors -- those nibbles moved
    to nibbles 0..3 -- are paired into four virtual lanes V = g // 2 (lane
    2V in bits 0..15, lane 2V+1 in bits 16..31) stored as quartets, word k
    of V at index 8 nf b + 4 k + V.
  The partial chunk takes 2 r b words, so the tile is dense.
V tile (1024 * v_avg_bits bytes): the 8 dim-tiles' quartets in order.
"""
import functools

import numpy as np

TILE = 64
V_MEMBERS = (0, 1, 8, 9)          # token offsets 2t + V_MEMBERS[n % 4]
HALF_NIBBLES = (0, 1, 4, 5)       # the real nibbles of a half quad


def _quartet_source(b, k, p):
    """(selector index s, nibble n, code bit) stored at bit p of plane word k."""
    n, q = p // 4, p % 4
    if b == 4:
        return k, n, q
    if b == 1:
        return q, n, 0
    if k < 2:                      # A (s0, s1) or B (s2, s3): the low two code bits
        return 2 * k + q // 2, n, q % 2
    return q, n, 2                 # H: bit 2 of s0..s3


def _k_selector_member(mu, j, lane, n):
    g, t = lane // 4, lane % 4
    return 16 * mu + g + 8 * (n >= 4), 16 * j + 4 * t + (n % 4)


def _v_selector_member(m, kappa, lane, n):
    g, t = lane // 4, lane % 4
    return 16 * kappa + 2 * t + V_MEMBERS[n % 4], 16 * m + g + 8 * (n >= 4)


@functools.lru_cache(maxsize=None)
def k_tile_bitmap(group_spec):
    """Source of every bit of a K tile.

    group_spec: tuple of (width, size) per group in record order.  Returns
    int arrays (token, position, code_bit), one entry per tile bit (bit q of
    32-bit word w is entry 32 w + q); every bit of the tile holds a code bit.
    """
    tok, pos, cb = [], [], []
    start = 0
    for b, d in group_spec:
        n_full = d // 16
        for j in range(n_full):
            for k in range(b):
                for lane in range(32):
                    for p in range(32):
                        s, n, bit = _quartet_source(b, k, p)
                        token, coord = _k_selector_member(s, j, lane, n)
                        tok.append(token)
                        pos.append(start + coord)
                        cb.append(bit)
        r = d - 16 * n_full
        if r:
            nf = r // 4
            for k in range(b):
                for g in range(8):
                    for t in range(nf):
                        for p in range(32):
                            s, n, bit = _quartet_source(b, k, p)
                            token, coord = _k_selector_member(s, n_full, 4 * g + t, n)
                            tok.append(token)
                            pos.append(start + coord)
                            cb.append(bit)
            if r % 4:
                for k in range(b):
                    for v in range(4):
                        for p in range(32):
                            s, nv, bit = _quartet_source(b, k, p)
                            g = 2 * v + nv // 4
                            n = HALF_NIBBLES[nv % 4]
                            token, coord = _k_selector_member(s, n_full, 4 * g + nf, n)
                            assert coord < d
                            tok.append(token)
                            pos.append(start + coord)
                            cb.append(bit)
        start += d
    return np.array(tok), np.array(pos), np.array(cb)


@functools.lru_cache(maxsize=None)
def v_tile_bitmap(vb):
    tok, pos, cb = [], [], []
    for m in range(8):
        for k in range(vb):
            for lane in range(32):
                for p in range(32):
                    s, n, bit = _quartet_source(vb, k, p)
                    token, coord = _v_selector_member(m, s, lane, n)
                    tok.append(token)
                    pos.append(coord)
                    cb.append(bit)
    return np.array(tok), np.array(pos), np.array(cb)


def _pack(codes, bitmap, nbytes):
    """codes int [tiles, 64, P] -> uint8 [tiles, nbytes] through a bit map."""
    tok, pos, cb = bitmap
    assert len(tok) == 8 * nbytes
    codes = np.asarray(codes, dtype=np.int64)
    bits = ((codes[:, tok, pos] >> cb[None, :]) & 1).astype(np.uint8)
    return np.packbits(bits, axis=1, bitorder="little")


def _inverse(bitmap, npos):
    """inv[token, position, code_bit] = the tile bit holding it (-1 if none)."""
    tok, pos, cb = bitmap
    inv = np.full((TILE, npos, 4), -1, dtype=np.int64)
    inv[tok, pos, cb] = np.arange(len(tok))
    return inv


def _unpack(tiles, bitmap, npos):
    """uint8 [tiles, nbytes] -> codes [tiles, 64, npos]: gather each code's bits."""
    inv = _inverse(bitmap, npos)
    tiles = np.asarray(tiles, dtype=np.uint8)
    bits = np.unpackbits(tiles, axis=1, bitorder="little")
    out = np.zeros((tiles.shape[0], TILE, npos), dtype=np.int64)
    for k in range(4):
        have = inv[:, :, k] >= 0
        idx = np.where(have, inv[:, :, k], 0)
        out += (bits[:, idx].astype(np.int64) * have[None]) << k
    return out


def stored_symbol(codes, b):
    """Codes -> the symbols a selector holds at width b (sigma at width 4)."""
    c = np.asarray(codes, dtype=np.int64)
    if b != 4:
        return c
    return np.where(c >= 8, c - 8, 15 - c)


def code_of_symbol(symbols, b):
    """Inverse of stored_symbol."""
    s = np.asarray(symbols, dtype=np.int64)
    if b != 4:
        return s
    return np.where(s >= 8, 15 - s, s + 8)


def _k_symbols(codes, groups, inverse=False):
    """Record-order K codes <-> symbols, group by group."""
    out = np.array(codes, dtype=np.int64, copy=True)
    start = 0
    for b, d in groups:
        cols = slice(start, start + len(d))
        out[..., cols] = (code_of_symbol if inverse else stored_symbol)(out[..., cols], int(b))
        start += len(d)
    return out


def group_spec(groups):
    """(width, size) tuple from oracle group layouts [(width, dims), ...]."""
    return tuple((int(b), len(d)) for b, d in groups)


def pack_k_tiles(codes, groups, k_avg_bits):
    """Record-order K codes [n, P] -> uint8 [ceil(n/64), 1024*k_avg_bits]; rows past n are code 0."""
    return _pack(_to_tiles(_k_symbols(codes, groups)), k_tile_bitmap(group_spec(groups)), 1024 * k_avg_bits)


def unpack_k_tiles(tiles, groups, n=None):
    sym = _unpack(tiles, k_tile_bitmap(group_spec(groups)), sum(len(d) for _, d in groups))
    codes = _k_symbols(sym.reshape(-1, sym.shape[-1]), groups, inverse=True)
    return codes if n is None else codes[:n]


def pack_v_tiles(codes, vb):
    return _pack(_to_tiles(stored_symbol(codes, vb)), v_tile_bitmap(vb), 1024 * vb)


def unpack_v_tiles(tiles, vb, n=None):
    codes = code_of_symbol(_unpack(tiles, v_tile_bitmap(vb), 128).reshape(-1, 128), vb)
    return codes if n is None else codes[:n]


def _to_tiles(codes):
    codes = np.asarray(codes, dtype=np.int64)
    n, p = codes.shape
    nt = (n + TILE - 1) // TILE
    out = np.zeros((nt * TILE, p), dtype=np.int64)
    out[:n] = codes
    return out.reshape(nt, TILE, p)


def quartet_pack(sel, b):
    """The plane words of one lane's quartet (reference form of the table above)."""
    s0, s1, s2, s3 = (int(x) for x in sel)
    m1, m3, m4 = 0x11111111, 0x33333333, 0x44444444
    if b == 4:
        return [s0, s1, s2, s3]
    if b == 1:
        return [((s0 & m1) | (s1 & m1) << 1 | (s2 & m1) << 2 | (s3 & m1) << 3) & 0xFFFFFFFF]
    a = ((s0 & m3) | (s1 & m3) << 2) & 0xFFFFFFFF
    bb = ((s2 & m3) | (s3 & m3) << 2) & 0xFFFFFFFF
    if b == 2:
        return [a, bb]
    h = ((s0 & m4) >> 2 | (s1 & m4) >> 1 | (s2 & m4) | (s3 & m4) << 1) & 0xFFFFFFFF
    return [a, bb, h]
