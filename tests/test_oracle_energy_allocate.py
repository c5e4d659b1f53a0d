"""Pins for oracle/energy.py and oracle/allocate.py."""
import itertools

import numpy as np
import pytest

from oracle import allocate as alloc
from oracle import energy
from oracle.lloyd_max import DISTORTION


def _brute_energy(q, k, pairing):
    """Plain Python-int loops over every element (fp16 -> exact int * 2**24)."""
    nq, hq, d = q.shape
    _, hkv, _ = k.shape
    g = hq // hkv
    blocks = energy.block_dims(d, pairing)
    eq = [[0] * len(blocks) for _ in range(hkv)]
    ek = [[0] * len(blocks) for _ in range(hkv)]
    for h in range(hkv):
        for j, (a, b) in enumerate(blocks):
            for r in range(nq):
                for hh in range(h * g, (h + 1) * g):
                    for dim in (a, b):
                        v = int(float(q[r, hh, dim]) * (1 << 24))
                        eq[h][j] += v * v
            for r in range(k.shape[0]):
                for dim in (a, b):
                    v = int(float(k[r, h, dim]) * (1 << 24))
                    ek[h][j] += v * v
    return eq, ek


@pytest.mark.parametrize("pairing", [0, 1])
def test_energy_exact_against_brute_force(pairing):
    rng = np.random.default_rng(pairing)
    q = (rng.standard_normal((5, 4, 16)) * np.exp(3 * rng.standard_normal(16))).astype(np.float16)
    k = (rng.standard_normal((7, 2, 16)) * np.exp(3 * rng.standard_normal(16))).astype(np.float16)
    # extremes: largest finite, smallest subnormal, zero, negative zero
    q[0, 0, :4] = [65504, -65504, 2.0 ** -24, -0.0]
    k[0, 1, :3] = [-65504, 2.0 ** -24, 6.1e-5]
    assert energy.block_energies(q, k, pairing) == _brute_energy(q, k, pairing)


def test_block_dims_pairings():
    assert energy.block_dims(8, 0) == [(0, 4), (1, 5), (2, 6), (3, 7)]
    assert energy.block_dims(8, 1) == [(0, 1), (2, 3), (4, 5), (6, 7)]


def test_scores_are_rope_invariant():
    """A RoPE rotation turns each block's 2-vector by an angle, so ||q_j|| and
    ||k_j|| (hence the score) do not change beyond fp16 rounding."""
    rng = np.random.default_rng(3)
    d, n = 128, 64
    sig = np.exp(rng.standard_normal(d // 2))
    x = rng.standard_normal((n, 1, d)) * np.concatenate([sig, sig])
    theta = 10000.0 ** (-np.arange(d // 2) * 2.0 / d)
    ang = np.arange(n)[:, None] * theta[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = x[..., : d // 2], x[..., d // 2:]
    xr = np.concatenate([a * c - b * s, a * s + b * c], axis=-1)
    e0 = np.array(energy.block_energies(x.astype(np.float16), x.astype(np.float16), 0)[0], dtype=float)
    e1 = np.array(energy.block_energies(xr.astype(np.float16), xr.astype(np.float16), 0)[0], dtype=float)
    assert np.allclose(e0, e1, rtol=3e-3)


def _brute_allocation_costs(scores, budget, b_min, b_max):
    best = None
    opt = []
    for w in itertools.product(range(b_min, b_max + 1), repeat=len(scores)):
        if sum(w) != budget:
            continue
        cost = sum(s * DISTORTION[b] for s, b in zip(scores, w))
        if best is None or cost < best - 1e-12 * abs(best):
            best, opt = cost, [w]
        elif abs(cost - best) <= 1e-12 * abs(best):
            opt.append(w)
    return best, opt


@pytest.mark.parametrize("seed", range(40))
def test_greedy_equals_brute_force_d8(seed):
    """D = 8 (four RoPE blocks): marginal-gain greedy over a convex distortion
    reaches the minimum of sum_j s_j Dist(b_j) found by exhaustive search."""
    rng = np.random.default_rng(seed)
    scores = np.exp(2.0 * rng.standard_normal(4))
    if seed % 5 == 0:
        scores[1] = scores[2]                  # exercise ties
    b_min = 0 if seed % 4 == 0 else 1
    for avg in range(b_min, 5):
        w = alloc.greedy_allocate(scores, avg, b_min, 4)
        best, opt = _brute_allocation_costs(scores, avg * 4, b_min, 4)
        cost = sum(s * DISTORTION[int(b)] for s, b in zip(scores, w))
        assert cost == pytest.approx(best, rel=1e-12)
        assert tuple(int(b) for b in w) in opt


def test_constant_scores_give_uniform_allocation():
    for avg in (1, 2, 3, 4):
        assert np.all(alloc.greedy_allocate(np.full(64, 2.5), avg) == avg)


def test_zero_scores_fill_lowest_blocks_first():
    """All gains are exactly 0: the tie rule (lower index) decides every step."""
    w = alloc.greedy_allocate(np.zeros(64), 2)
    assert list(w) == [4] * 21 + [2] + [1] * 42


def test_ties_go_to_lower_index_and_monotone():
    w = alloc.greedy_allocate([1.0, 1.0, 1.0, 1.0], 2, 1, 4)       # budget 8: +1 to each
    assert list(w) == [2, 2, 2, 2]
    w = alloc.greedy_allocate([1.0, 1.0, 1.0, 1.0], 1, 0, 4)       # budget 4 from 0
    assert list(w) == [1, 1, 1, 1]
    w = alloc.greedy_allocate([1.0, 1.0, 1.0], 1, 1, 4)
    assert list(w) == [1, 1, 1]
    w = alloc.greedy_allocate([3.0, 3.0, 0.5, 0.1], 2, 1, 4)
    assert list(w) == [3, 3, 1, 1]
    rng = np.random.default_rng(1)
    s = np.exp(2 * rng.standard_normal(64))
    w = alloc.greedy_allocate(s, 3)
    order = np.argsort(-s, kind="stable")
    assert np.all(np.diff(w[order]) <= 0)          # more energy never gets fewer bits
    assert w.sum() == 192 and w.min() >= 1 and w.max() <= 4


def test_group_layout():
    bw = np.array([3, 1, 4, 3])
    groups = alloc.group_layout(bw, 8, 0)
    assert [b for b, _ in groups] == [4, 3, 1]
    assert [list(d) for _, d in groups] == [[2, 6], [0, 3, 4, 7], [1, 5]]
    groups = alloc.group_layout(np.array([0, 2, 2, 0]), 8, 1)
    assert [(b, list(d)) for b, d in groups] == [(2, [2, 3, 4, 5])]
