"""Pins of the oracle's per-layer logit MAE (Block-GTQ abstract: per-layer MAE
of the RoPE query-key logits; blockgtq README, bit allocation: the per-layer
kernel MAE against uniform TQ-MSE)."""
import numpy as np
import pytest
import torch

from oracle import diag, model
from oracle.attention import dequantise_keys
from oracle import tiles
from packed_decode_attention_b200 import workloads as wl

# N(0,1) Lloyd-Max mean squared errors per coordinate (Max 1960, Table I)
D_B = {1: 0.363380, 2: 0.117482, 3: 0.034548, 4: 0.009497}


def _uniform(bits, seed=11, g=4):
    cfg = model.Config(1, 1, g, 128, bits, 3, 1, 4, 0, seed)
    return model.Tables(cfg, np.full((1, 1, 64), bits))


@pytest.mark.parametrize("bits,m", [(1, 256), (2, 384), (3, 384), (4, 256)])
def test_gaussian_keys_closed_form(bits, m):
    """Keys and queries N(0, I): with one group of all 128 dims the key error
    e has E|e|^2 ~= D * D(b) (TQ-MSE on u = sqrt(d) R k / |k|), and q . e is
    N(0, |e|^2) given e, so E|q . e| / sqrt(D) ~= sqrt(2/pi * D(b)).  u's
    coordinates follow the sphere's marginal, slightly lighter-tailed than
    N(0,1), which puts the oracle a little (< 3 %) below the Gaussian figure."""
    rng = np.random.default_rng(100 + bits)
    tb = _uniform(bits)
    k = rng.standard_normal((m, 128)).astype(np.float16)
    q = rng.standard_normal((m, 4, 128)).astype(np.float16)
    enc = model.encode_rows(tb, 0, 0, k, k)
    mae = diag.logit_mae(tb, 0, 0, q, k, enc["k_tiles"], enc["k_norms"])
    ratio = mae.mean() / np.sqrt(2.0 / np.pi * D_B[bits])
    assert 0.96 < ratio < 1.01, ratio


def test_brute_force_tiny():
    """Every causal pair by explicit loops over pairs and coordinates."""
    rng = np.random.default_rng(3)
    tb = _uniform(2, g=2)
    m = 5
    k = (rng.standard_normal((m, 128)) * 2).astype(np.float16)
    q = rng.standard_normal((m, 2, 128)).astype(np.float16)
    enc = model.encode_rows(tb, 0, 0, k, k)
    got = diag.logit_mae(tb, 0, 0, q, k, enc["k_tiles"], enc["k_norms"])
    groups = tb.groups[0, 0]
    k_hat = dequantise_keys(tiles.unpack_k_tiles(enc["k_tiles"], groups, m), enc["k_norms"], groups, tb.k_rot[0, 0],
                            tb.codebooks, 128)
    want = []
    for h in range(2):
        total, pairs = 0.0, 0
        for i in range(m):
            for j in range(i + 1):
                s = 0.0
                for d in range(128):
                    s += float(q[i, h, d]) * (float(k[j, d]) - k_hat[j, d])
                total += abs(s) / np.sqrt(128.0)
                pairs += 1
        want.append(total / pairs)
    assert pairs == diag.causal_pair_count(m) == 15
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=0)


def _setup(m=64, seed=5):
    rng = np.random.default_rng(seed)
    tb = _uniform(3, g=2)
    k = rng.standard_normal((m, 128)).astype(np.float16)
    q = rng.standard_normal((m, 2, 128)).astype(np.float16)
    return tb, k, q


def test_scaling_and_zero_query():
    tb, k, q = _setup()
    enc = model.encode_rows(tb, 0, 0, k, k)
    a = diag.logit_mae(tb, 0, 0, q, k, enc["k_tiles"], enc["k_norms"])
    b = diag.logit_mae(tb, 0, 0, (q.astype(np.float32) * 2).astype(np.float16), k, enc["k_tiles"], enc["k_norms"])
    np.testing.assert_allclose(b, 2 * a, rtol=1e-13)
    z = diag.logit_mae(tb, 0, 0, np.zeros_like(q), k, enc["k_tiles"], enc["k_norms"])
    assert np.all(z == 0)


def test_last_key_enters_one_pair():
    """Key M-1 is seen only by query M-1: changing it moves the MAE by that
    one pair's change / (M (M + 1) / 2).  A transposed mask would count it M
    times."""
    tb, k, q = _setup()
    m = k.shape[0]
    enc = model.encode_rows(tb, 0, 0, k, k)
    a = diag.logit_mae(tb, 0, 0, q, k, enc["k_tiles"], enc["k_norms"])
    k2 = k.copy()
    k2[m - 1] = (k2[m - 1].astype(np.float32) * -3).astype(np.float16)
    enc2 = model.encode_rows(tb, 0, 0, k2, k2)
    b = diag.logit_mae(tb, 0, 0, q, k2, enc2["k_tiles"], enc2["k_norms"])
    groups = tb.groups[0, 0]

    def last_pair(kk, e):
        kh = dequantise_keys(tiles.unpack_k_tiles(e["k_tiles"], groups, m), e["k_norms"], groups, tb.k_rot[0, 0],
                             tb.codebooks, 128)[m - 1]
        return np.abs(q[m - 1].astype(np.float64) @ (kk[m - 1].astype(np.float64) - kh)) / np.sqrt(128.0)

    np.testing.assert_allclose(b - a, (last_pair(k2, enc2) - last_pair(k, enc)) / diag.causal_pair_count(m),
                               rtol=1e-9, atol=1e-15)


def test_window_offset_equals_fresh_cache():
    """TQ-MSE encodes each row on its own, so the window [w0, w0 + M) of a
    longer cache gives the MAE of a cache holding only those rows."""
    rng = np.random.default_rng(9)
    tb = _uniform(3, g=2)
    k = rng.standard_normal((150, 128)).astype(np.float16)
    q = rng.standard_normal((70, 2, 128)).astype(np.float16)
    enc = model.encode_rows(tb, 0, 0, k, k)
    a = diag.logit_mae(tb, 0, 0, q, k[80:150], enc["k_tiles"], enc["k_norms"], w0=80)
    enc2 = model.encode_rows(tb, 0, 0, k[80:150], k[80:150])
    b = diag.logit_mae(tb, 0, 0, q, k[80:150], enc2["k_tiles"], enc2["k_norms"])
    np.testing.assert_array_equal(a, b)


def test_block_gtq_beats_uniform_on_uneven_energies():
    """The pages' claim in synthetic form: with log-normal per-block energies
    (shape 1), the energy-driven allocation lowers the logit MAE of every
    (layer, KV head) against uniform TQ-MSE at the same 3-bit average."""
    w = wl.scaled(wl.WORKLOADS["qwen3b"], n_layers=3, seq_len=256, n_calib=256)
    cfg = model.Config(w.n_layers, w.n_kv_heads, w.n_q_heads, 128, 3, 3, 1, 4, 0, w.seed)
    cq, ck = wl.calibration(w)
    gtq = model.Tables(cfg, model.allocate(cfg, cq.numpy(), ck.numpy()))
    uni = model.Tables(cfg, np.full((w.n_layers, w.n_kv_heads, 64), 3))
    m = 128
    for layer in range(w.n_layers):
        k = wl.keys(w, layer, 0, 0, m).numpy()
        q = wl.queries(w, layer, 0, torch.arange(m), tag=3).numpy()
        for h in range(w.n_kv_heads):
            qh = q[:, h * w.group:(h + 1) * w.group]
            res = []
            for tb in (gtq, uni):
                enc = model.encode_rows(tb, layer, h, k[:, h], k[:, h])
                res.append(diag.logit_mae(tb, layer, h, qh, k[:, h], enc["k_tiles"], enc["k_norms"]).mean())
            assert res[0] < res[1], (layer, h, res)
