"""Pins for oracle/tiles.py: the tile format's two renderings agree, it is a
bijection on codes, and a hand-worked quartet."""
import numpy as np
import pytest

from oracle import allocate as oalloc
from oracle import tiles


def test_quartet_golden(golden):
    for row in golden("quartet_example.txt"):
        b = int(row[0])
        sel = [int(x, 16) for x in row[1:5]]
        assert [f"{w:08X}" for w in tiles.quartet_pack(sel, b)] == row[5:]


def _symbol(c, b):
    """The stored symbol of code c at width b, from its definition: widths 1..3
    store c; width 4 stores the sign of the level in bit 3 and the rank of
    |level| among the positive levels in bits 0..2."""
    if b != 4:
        return int(c)
    negative = c < 8
    rank = (7 - c) if negative else (c - 8)     # C[c] = -C[15 - c]: |C[c]| = C[8 + rank]
    return (8 if negative else 0) | rank


def _selectors_k(codes_tile, start, d, j, lane, b):
    """Lane's four selector words for chunk j from the plain definition
    (nibbles whose coordinate is past the group are 0)."""
    out = []
    for mu in range(4):
        w = 0
        for n in range(8):
            token, coord = tiles._k_selector_member(mu, j, lane, n)
            if coord < d:
                w |= _symbol(codes_tile[token, start + coord], b) << (4 * n)
        out.append(w)
    return out


@pytest.mark.parametrize("widths_seed", range(6))
def test_k_tile_quartets_match_the_plane_formulas(widths_seed):
    rng = np.random.default_rng(widths_seed)
    kavg = 2 + widths_seed % 2
    bw = np.full(64, kavg)
    idx = rng.permutation(64)
    for a, c in zip(idx[:25], idx[25:50]):            # move bits, keeping the budget
        if bw[a] < 4 and bw[c] > 1:
            bw[a] += 1
            bw[c] -= 1
    groups = oalloc.group_layout(bw, 128, 0)
    assert any(len(d) % 16 for _, d in groups) or widths_seed > 3
    codes = np.concatenate([rng.integers(0, 1 << b, size=(64, len(d))) for b, d in groups], axis=1)
    packed = tiles.pack_k_tiles(codes, groups, kavg)[0]
    words = packed.view("<u4")
    assert len(words) == 256 * kavg
    off = 0
    start = 0
    for b, d in groups:
        d = len(d)
        for j in range(d // 16):
            for lane in range(32):
                expect = tiles.quartet_pack(_selectors_k(codes, start, d, j, lane, b), b)
                got = [int(words[off + 32 * k + lane]) for k in range(b)]
                assert got == expect, (b, d, j, lane)
            off += 32 * b
        r = d % 16
        if r:
            j = d // 16
            nf = r // 4
            for g in range(8):
                for t in range(nf):
                    expect = tiles.quartet_pack(_selectors_k(codes, start, d, j, 4 * g + t, b), b)
                    got = [int(words[off + 8 * nf * k + g * nf + t]) for k in range(b)]
                    assert got == expect, ("partial full lane", b, d, g, t)
            if r % 4:
                for v in range(4):
                    halves = []
                    for g in (2 * v, 2 * v + 1):
                        sel = _selectors_k(codes, start, d, j, 4 * g + nf, b)       # padding nibbles are 0
                        halves.append([(w & 0xFF) | ((w >> 8) & 0xFF00) for w in sel])
                    virt = [halves[0][mu] | (halves[1][mu] << 16) for mu in range(4)]
                    got = [int(words[off + 8 * nf * b + 4 * k + v]) for k in range(b)]
                    assert got == tiles.quartet_pack(virt, b), ("partial half lanes", b, d, v)
            off += 2 * r * b
        start += d
    assert off == len(words)


@pytest.mark.parametrize("seed", range(4))
def test_round_trips(seed):
    rng = np.random.default_rng(seed)
    for _ in range(3):
        bw = np.full(64, 3)
        idx = rng.permutation(64)
        # move bits between blocks keeping the sum (widths 1..4)
        for a, c in zip(idx[:20], idx[20:40]):
            if bw[a] < 4 and bw[c] > 1:
                bw[a] += 1
                bw[c] -= 1
        groups = oalloc.group_layout(bw, 128, 0)
        n = int(rng.integers(1, 300))
        codes = np.concatenate([rng.integers(0, 1 << b, size=(n, len(d))) for b, d in groups], axis=1)
        t = tiles.pack_k_tiles(codes, groups, 3)
        assert t.shape == ((n + 63) // 64, 3072)
        assert np.array_equal(tiles.unpack_k_tiles(t, groups, n), codes)
        for vb in (1, 2, 3, 4):
            vc = rng.integers(0, 1 << vb, size=(n, 128))
            vt = tiles.pack_v_tiles(vc, vb)
            assert vt.shape == ((n + 63) // 64, 1024 * vb)
            assert np.array_equal(tiles.unpack_v_tiles(vt, vb, n), vc)


def test_v_tile_layout_matches_fragment_order():
    """Word (m, k, lane) holds plane k of the lane's quartet for dim-tile m."""
    rng = np.random.default_rng(9)
    vc = rng.integers(0, 8, size=(64, 128))
    words = tiles.pack_v_tiles(vc, 3)[0].view("<u4")
    for m in (0, 5, 7):
        for lane in (0, 13, 31):
            sel = []
            for kappa in range(4):
                w = 0
                for n in range(8):
                    token, coord = tiles._v_selector_member(m, kappa, lane, n)
                    w |= int(vc[token, coord]) << (4 * n)
                sel.append(w)
            assert [int(words[m * 96 + 32 * k + lane]) for k in range(3)] == tiles.quartet_pack(sel, 3)


def test_every_code_bit_stored_once():
    groups = oalloc.group_layout(np.array([4] * 10 + [3] * 30 + [2] * 14 + [1] * 10), 128, 0)
    tok, pos, cb = tiles.k_tile_bitmap(tiles.group_spec(groups))
    widths = np.concatenate([np.full(len(d), b) for b, d in groups])
    keys = set(zip(tok.tolist(), pos.tolist(), cb.tolist()))
    assert len(keys) == len(tok) == 64 * int(widths.sum())
    assert all(c < widths[p] for _, p, c in keys)


def test_width4_symbols_stand_for_their_levels():
    """Symbol s of a width-4 code is the level's sign (bit 3) and the rank of
    |level| (bits 0..2): the stored symbol maps every code to a distinct
    symbol, the inverse undoes it, and with the binary16 Lloyd-Max table the
    level read back by sign and magnitude is the code's own level."""
    from oracle import lloyd_max as lm
    c16, _ = lm.codebook_fp16(4)
    codes = np.arange(16)
    sym = tiles.stored_symbol(codes, 4)
    assert sorted(sym.tolist()) == list(range(16))
    assert np.array_equal(tiles.code_of_symbol(sym, 4), codes)
    for c, s in zip(codes, sym):
        assert s == _symbol(c, 4)
        level = (-1.0 if s >= 8 else 1.0) * c16[8 + (s & 7)]
        assert level == c16[c]
    for b in (1, 2, 3):
        assert np.array_equal(tiles.stored_symbol(np.arange(1 << b), b), np.arange(1 << b))


def test_v_tile_width4_holds_symbols():
    rng = np.random.default_rng(11)
    vc = rng.integers(0, 16, size=(64, 128))
    words = tiles.pack_v_tiles(vc, 4)[0].view("<u4")
    m, lane = 3, 17
    for kappa in range(4):
        w = 0
        for n in range(8):
            token, coord = tiles._v_selector_member(m, kappa, lane, n)
            w |= _symbol(vc[token, coord], 4) << (4 * n)
        assert int(words[m * 128 + 32 * kappa + lane]) == w
