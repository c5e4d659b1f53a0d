"""Pins for oracle/rope.py and the fused RoPE + encode of oracle/model.py:
hand-worked rotations for both pairings, the identity at position 0, the
norm of every block kept, composition of positions, the relative-position
property of RoPE logits, agreement with the rotate_half formulation, and the
fused encode's invariants."""
import numpy as np
import pytest

from oracle import model, rope


def test_hand_worked_half_split():
    # D = 4, half-split: blocks (0, 2) with theta 1 and (1, 3) with theta base^(-1/2)
    out = rope.apply_rope(np.array([[1.0, 0.0, 0.0, 0.0]]), [1], 10000.0, pairing=0)
    np.testing.assert_allclose(out, [[np.cos(1.0), 0.0, np.sin(1.0), 0.0]], atol=1e-15)
    out = rope.apply_rope(np.array([[0.0, 1.0, 0.0, 0.0]]), [100], 10000.0, pairing=0)  # 100 * 0.01 = 1 rad
    np.testing.assert_allclose(out, [[0.0, np.cos(1.0), 0.0, np.sin(1.0)]], atol=1e-14)
    out = rope.apply_rope(np.array([[0.0, 0.0, 1.0, 0.0]]), [1], 10000.0, pairing=0)
    np.testing.assert_allclose(out, [[-np.sin(1.0), 0.0, np.cos(1.0), 0.0]], atol=1e-15)


def test_hand_worked_interleaved():
    out = rope.apply_rope(np.array([[1.0, 0.0, 0.0, 0.0]]), [1], 10000.0, pairing=1)
    np.testing.assert_allclose(out, [[np.cos(1.0), np.sin(1.0), 0.0, 0.0]], atol=1e-15)
    out = rope.apply_rope(np.array([[0.0, 0.0, 0.0, 1.0]]), [100], 10000.0, pairing=1)
    np.testing.assert_allclose(out, [[0.0, 0.0, -np.sin(1.0), np.cos(1.0)]], atol=1e-14)


def test_inverse_frequencies():
    th = rope.inv_freq(128, 1e6)
    assert th[0] == 1.0 and len(th) == 64
    np.testing.assert_allclose(th[32], 1e6 ** -0.5, rtol=1e-15)
    np.testing.assert_allclose(th[1:] / th[:-1], 1e6 ** (-2.0 / 128), rtol=1e-13)


@pytest.mark.parametrize("pairing", [0, 1])
def test_position_zero_is_identity_and_block_norms_are_kept(pairing):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 128))
    assert np.array_equal(rope.apply_rope(x, np.zeros(6), 1e6, pairing), x)
    pos = rng.integers(0, 1 << 20, 6)
    y = rope.apply_rope(x, pos, 1e6, pairing)
    if pairing == 0:
        nx = x[:, :64] ** 2 + x[:, 64:] ** 2
        ny = y[:, :64] ** 2 + y[:, 64:] ** 2
    else:
        nx = x[:, 0::2] ** 2 + x[:, 1::2] ** 2
        ny = y[:, 0::2] ** 2 + y[:, 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12)


@pytest.mark.parametrize("pairing", [0, 1])
def test_positions_compose_and_logits_depend_on_the_offset(pairing):
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, 128))
    a, b = rng.integers(0, 5000, 5), rng.integers(0, 5000, 5)
    np.testing.assert_allclose(rope.apply_rope(rope.apply_rope(x, a, 1e4, pairing), b, 1e4, pairing),
                               rope.apply_rope(x, a + b, 1e4, pairing), atol=1e-9)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    m, n, s = 700, 123, 4096
    l1 = rope.apply_rope(q[None], [m], 1e4, pairing)[0] @ rope.apply_rope(k[None], [n], 1e4, pairing)[0]
    l2 = rope.apply_rope(q[None], [m + s], 1e4, pairing)[0] @ rope.apply_rope(k[None], [n + s], 1e4, pairing)[0]
    np.testing.assert_allclose(l1, l2, rtol=1e-9, atol=1e-9)


def test_matches_the_rotate_half_formulation():
    # x * cos + rotate_half(x) * sin, rotate_half(x) = (-x2, x1), angles repeated over the halves
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 128))
    pos = np.array([0, 1, 4097, 131071])
    ang = pos[:, None] * (1e6 ** (-np.arange(0, 128, 2) / 128.0))[None, :]
    cos = np.concatenate([np.cos(ang), np.cos(ang)], axis=1)
    sin = np.concatenate([np.sin(ang), np.sin(ang)], axis=1)
    rot = np.concatenate([-x[:, 64:], x[:, :64]], axis=1)
    np.testing.assert_allclose(rope.apply_rope(x, pos, 1e6, 0), x * cos + rot * sin, atol=1e-12)


def _tables(seed=7):
    cfg = model.Config(n_layers=1, n_kv_heads=1, n_q_heads=4, head_dim=128, k_avg_bits=3, v_avg_bits=3,
                       b_min=1, b_max=4, pairing=0, seed=seed)
    rng = np.random.default_rng(seed)
    widths = np.full((1, 1, 64), 3, dtype=np.int64)
    widths[0, 0, :8] = 4
    widths[0, 0, 8:16] = 2
    return model.Tables(cfg, widths), rng


def test_fused_encode_at_position_zero_is_the_plain_encode():
    tb, rng = _tables()
    k = rng.standard_normal((70, 128)).astype(np.float16)
    v = rng.standard_normal((70, 128)).astype(np.float16)
    a = model.encode_rows(tb, 0, 0, k, v)
    b = model.encode_rows_rope(tb, 0, 0, k, v, np.zeros(70, dtype=np.int64), 1e6)
    for key in ("k_tiles", "k_norms", "v_tiles", "v_norm"):
        assert np.array_equal(a[key], b[key]), key


def test_fused_encode_keeps_group_norms_and_matches_rope_then_encode():
    """Groups hold whole RoPE blocks, so the fused encode's norms are the
    pre-RoPE norms; its codes match encoding fp16(RoPE(k)) except where that
    rounding moves u across a threshold."""
    tb, rng = _tables(8)
    n = 200
    k = (rng.standard_normal((n, 128)) * np.exp(rng.standard_normal(128))).astype(np.float16)
    v = rng.standard_normal((n, 128)).astype(np.float16)
    pos = np.arange(5000, 5000 + n)
    fused = model.encode_rows_rope(tb, 0, 0, k, v, pos, 1e6)
    plain = model.encode_rows(tb, 0, 0, k, v)
    assert np.array_equal(fused["k_norms"], plain["k_norms"])      # RoPE keeps every block's norm
    assert np.array_equal(fused["v_tiles"], plain["v_tiles"])       # values are not turned
    k_rot = rope.apply_rope(k.astype(np.float64), pos, 1e6, 0).astype(np.float16)
    ref = model.encode_rows(tb, 0, 0, k_rot, v)
    agree = np.mean(fused["k_codes"] == ref["k_codes"])
    assert agree > 0.99, agree
    assert np.max(np.abs(fused["k_codes"] - ref["k_codes"])) <= 1
