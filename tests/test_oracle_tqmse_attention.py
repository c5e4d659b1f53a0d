"""Pins for oracle/tqmse.py, oracle/attention.py and oracle/model.py."""
import numpy as np
import pytest

from oracle import attention, haar, lloyd_max, model, tqmse


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_centroid_patterns_encode_back(bits):
    """A row whose rotated, normalised coordinates are sqrt(d) c / ||c|| for
    centroid values c encodes back to c's codes whenever that scaled pattern
    stays inside each centroid's cell (rows that would cross a threshold are
    dropped)."""
    d = 24
    rng = np.random.default_rng(bits)
    rot = haar.rotation_fp32(d, 9, 0, 0, 0, bits)
    cb, th = (a.astype(np.float64) for a in lloyd_max.codebook_fp16(bits))
    edges = np.concatenate(([-np.inf], th, [np.inf]))
    prob = np.diff([0.0] + [0.5 * (1 + __import__("math").erf(t / np.sqrt(2))) for t in th] + [1.0])
    codes = rng.choice(len(cb), p=prob, size=(400, d))
    c = cb[codes]
    f = np.sqrt(d) / np.linalg.norm(c, axis=1)
    u = f[:, None] * c
    inside = np.all((u > edges[codes] + 1e-4) & (u < edges[codes + 1] - 1e-4), axis=1)
    assert inside.sum() > 100
    scale = rng.uniform(0.1, 10.0, size=(400, 1))
    x = scale * (c @ np.linalg.inv(rot.astype(np.float64)).T)         # Pi x = scale * c
    got, norms = tqmse.encode_group(x, np.arange(d), rot, bits)
    assert np.array_equal(got[inside], codes[inside])
    assert np.allclose(norms, np.linalg.norm(x, axis=1), rtol=1e-12)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_u_mse_on_gaussian_rows_near_lloyd_max(bits):
    d = 128
    rng = np.random.default_rng(20 + bits)
    x = rng.standard_normal((3000, d))
    rot = haar.rotation_fp32(d, 1, 0, 0, 0, bits)
    codes, norms = tqmse.encode_group(x, np.arange(d), rot, bits)
    y = x @ rot.astype(np.float64).T
    u = np.sqrt(d) * y / norms[:, None]
    cb = lloyd_max.codebook_fp16(bits)[0].astype(np.float64)
    err = np.mean((u - cb[codes]) ** 2)
    # u is sqrt(d) times a uniform point on the sphere: close to N(0,1) at d = 128
    assert abs(err - lloyd_max.mse(bits)) < 0.03 * lloyd_max.mse(bits)


def test_zero_row_and_norm_rounding():
    cfg = model.Config(1, 1, 2, k_avg_bits=2, v_avg_bits=2, seed=3)
    bw = np.full((1, 1, 64), 2)
    bw[0, 0, :8] = 3
    bw[0, 0, 8:16] = 1
    tb = model.Tables(cfg, bw)
    k = np.zeros((2, 128), np.float16)
    v = np.zeros((2, 128), np.float16)
    k[1] = 1.0
    out = model.encode_rows(tb, 0, 0, k, v)
    assert np.all(out["k_codes"][0][:16] == 4) and np.all(out["k_codes"][0][16:128 - 16] == 2)
    assert np.all(out["k_norms"][0] == 0) and out["v_norm"][0] == 0
    # group norms of a row of ones: sqrt(d_g), rounded to fp16
    dg = [len(d) for _, d in tb.groups[0, 0]]
    assert list(out["k_norms"][1][:3].astype(np.float64)) == [float(np.float16(np.sqrt(x))) for x in dg]
    assert out["k_tiles"].shape == (1, 2048) and out["v_tiles"].shape == (1, 2048)


def _one_layer(seed=0, t=37, g=4, kb=3, vb=3):
    cfg = model.Config(1, 1, g, k_avg_bits=kb, v_avg_bits=vb, seed=seed)
    rng = np.random.default_rng(seed)
    cq = rng.standard_normal((1, 32, g, 128)).astype(np.float16)
    ck = (rng.standard_normal((1, 32, 1, 128)) * np.exp(rng.standard_normal(128))).astype(np.float16)
    tb = model.Tables(cfg, model.allocate(cfg, cq, ck))
    k = (rng.standard_normal((t, 128)) * np.exp(rng.standard_normal(128))).astype(np.float16)
    v = rng.standard_normal((t, 128)).astype(np.float16)
    enc = model.encode_rows(tb, 0, 0, k, v)
    q = rng.standard_normal((g, 128)).astype(np.float16)
    return cfg, tb, enc, q


def _dequant(tb, enc):
    kh = attention.dequantise_keys(enc["k_codes"], enc["k_norms"], tb.groups[0, 0], tb.k_rot[0, 0], tb.codebooks, 128)
    vh = attention.dequantise_values(enc["v_codes"], enc["v_norm"], tb.v_rot[0, 0], tb.codebooks[3], 128)
    return kh, vh


def _decode(tb, q, enc, n=None):
    n = enc["n"] if n is None else n
    return model.decode(tb, 0, 0, q, enc["k_tiles"], enc["k_norms"], enc["v_tiles"], enc["v_norm"], n)


def test_decode_single_token_returns_v_hat():
    cfg, tb, enc, q = _one_layer(t=1)
    _, vh = _dequant(tb, enc)
    out = _decode(tb, q, enc)
    assert np.allclose(out, np.repeat(vh, 4, axis=0), rtol=0, atol=1e-14)


def test_decode_equal_logits_give_mean():
    cfg, tb, enc, q = _one_layer()
    _, vh = _dequant(tb, enc)
    out = _decode(tb, np.zeros_like(q), enc)
    assert np.allclose(out, vh.mean(axis=0)[None, :], atol=1e-14)


def test_decode_empty_sequence_is_zero():
    cfg, tb, enc, q = _one_layer()
    out = _decode(tb, q, enc, n=0)
    assert np.all(out == 0)


def test_decode_dominant_token_and_permutation():
    cfg, tb, enc, q = _one_layer(t=20)
    kh, vh = _dequant(tb, enc)
    # a query parallel to one key, scaled up, puts all weight on it
    qd = np.repeat(kh[7:8] * 1e3 / np.linalg.norm(kh[7]), 4, axis=0)
    out = attention.attend(qd, kh, vh)
    assert np.allclose(out, vh[7][None, :], atol=1e-6)
    perm = np.random.default_rng(0).permutation(20)
    a = attention.attend(q.astype(np.float64), kh, vh)
    b = attention.attend(q.astype(np.float64), kh[perm], vh[perm])
    assert np.allclose(a, b, atol=1e-13)
    assert np.allclose(_decode(tb, q, enc), a, atol=1e-13)


def test_rotated_domain_logits_equal_dense_logits():
    """q . k_hat = sum_g n_g (q~_g . C[codes_g]) with q~ from rotated_query:
    the identity the GPU decode relies on (no orthogonality needed)."""
    cfg, tb, enc, q = _one_layer(t=50)
    kh, _ = _dequant(tb, enc)
    dense = q.astype(np.float64) @ kh.T / np.sqrt(128.0)
    qt = model.rotated_query(tb, 0, 0, q)
    codes = enc["k_codes"]
    rot = np.zeros_like(dense)
    pos = 0
    for gi, (b, dims) in enumerate(tb.groups[0, 0]):
        c = tb.codebooks[b].astype(np.float64)[codes[:, pos:pos + len(dims)]]
        n = enc["k_norms"][:, gi].astype(np.float64)
        rot += (qt[:, pos:pos + len(dims)] @ c.T) * n[None, :]
        pos += len(dims)
    assert np.allclose(rot, dense, rtol=1e-12, atol=1e-12)


def test_dequantised_keys_close_to_inputs():
    """Relative MSE of k_hat against k is about the Lloyd-Max distortion of the widths used."""
    cfg = model.Config(1, 1, 1, k_avg_bits=3, v_avg_bits=3, seed=5)
    tb = model.Tables(cfg, np.full((1, 1, 64), 3))
    rng = np.random.default_rng(5)
    k = rng.standard_normal((2000, 128)).astype(np.float16)
    enc = model.encode_rows(tb, 0, 0, k, k)
    kh, vh = _dequant(tb, enc)
    rel = np.sum((kh - k.astype(np.float64)) ** 2) / np.sum(k.astype(np.float64) ** 2)
    assert abs(rel - lloyd_max.mse(3)) < 0.05 * lloyd_max.mse(3)
    relv = np.sum((vh - k.astype(np.float64)) ** 2) / np.sum(k.astype(np.float64) ** 2)
    assert abs(relv - lloyd_max.mse(3)) < 0.05 * lloyd_max.mse(3)
