"""Pins of the oracle's buffered decode (the blockgtq README's "withbuffer"
setting: sink and recent-window positions kept in fp16 next to the packed
cache, one softmax over both)."""
import numpy as np
import pytest
import torch

from oracle import model
from packed_decode_attention_b200 import workloads as wl


@pytest.fixture(scope="module")
def setup():
    w = wl.scaled(wl.WORKLOADS["tiny"], seq_len=300, n_calib=64)
    cfg = model.Config(1, 1, 4, 128, 3, 3, 1, 4, 0, 7)
    cq, ck = wl.calibration(w)
    tb = model.Tables(cfg, model.allocate(cfg, cq.numpy(), ck.numpy()))
    k = wl.keys(w, 0, 0, 0, 300)[:, 0].numpy()
    v = wl.values(w, 0, 0, 0, 300)[:, 0].numpy()
    enc = model.encode_rows(tb, 0, 0, k, v)
    q = wl.decode_query(w, 0, [300])[0].numpy()
    return tb, enc, q, k, v


def _dec(tb, enc, q, lo, hi, bk, bv):
    return model.decode_buffered(tb, 0, 0, q, enc["k_tiles"], enc["k_norms"], enc["v_tiles"], enc["v_norm"], lo, hi,
                                 bk, bv)


def test_no_buffer_equals_decode(setup):
    tb, enc, q, k, v = setup
    empty = np.zeros((0, 128), dtype=np.float16)
    ref = model.decode(tb, 0, 0, q, enc["k_tiles"], enc["k_norms"], enc["v_tiles"], enc["v_norm"], 300)
    assert np.array_equal(_dec(tb, enc, q, 0, 300, empty, empty), ref)


def test_buffer_only_equals_library_attention(setup):
    """No packed position: plain softmax attention over the fp16 rows, checked
    against torch's scaled_dot_product_attention in float64."""
    tb, enc, q, k, v = setup
    got = _dec(tb, enc, q, 10, 10, k[:40], v[:40])
    qt = torch.from_numpy(q.astype(np.float64))[None, :, None, :]                     # [1, G, 1, D]
    kt = torch.from_numpy(k[:40].astype(np.float64))[None, None].expand(1, 4, 40, 128)
    vt = torch.from_numpy(v[:40].astype(np.float64))[None, None].expand(1, 4, 40, 128)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, :, 0].numpy()
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_buffer_rows_permute_freely(setup):
    tb, enc, q, k, v = setup
    rows = np.r_[0:4, 172:300]
    perm = np.random.default_rng(3).permutation(len(rows))
    a = _dec(tb, enc, q, 4, 172, k[rows], v[rows])
    b = _dec(tb, enc, q, 4, 172, k[rows][perm], v[rows][perm])
    assert np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(a))


def test_softmax_splits_at_the_packed_buffer_boundary(setup):
    """Attention over packed U buffer equals the log-sum-exp merge of the two
    parts attended separately (what the GPU's combine does)."""
    tb, enc, q, k, v = setup
    rows = np.r_[0:4, 172:300]
    whole = _dec(tb, enc, q, 4, 172, k[rows], v[rows])
    empty = np.zeros((0, 128), dtype=np.float16)
    # the two parts with their own softmax denominators, from the dequantised rows
    groups = tb.groups[0, 0]
    from oracle import tiles
    from oracle.attention import dequantise_keys, dequantise_values
    kc = tiles.unpack_k_tiles(enc["k_tiles"], groups, 172)[4:172]
    vc = tiles.unpack_v_tiles(enc["v_tiles"], 3, 172)[4:172]
    kh = dequantise_keys(kc, enc["k_norms"][4:172], groups, tb.k_rot[0, 0], tb.codebooks, 128)
    vh = dequantise_values(vc, enc["v_norm"][4:172], tb.v_rot[0, 0], tb.codebooks[3], 128)
    q64 = q.astype(np.float64)
    parts = []
    for kk, vv in ((kh, vh), (k[rows].astype(np.float64), v[rows].astype(np.float64))):
        lg = q64 @ kk.T / np.sqrt(128.0)
        m = lg.max(axis=1, keepdims=True)
        p = np.exp(lg - m)
        parts.append((m[:, 0], p.sum(axis=1), p @ vv))
    M = np.maximum(parts[0][0], parts[1][0])
    w = [np.exp(pm - M) for pm, _, _ in parts]
    merged = (w[0][:, None] * parts[0][2] + w[1][:, None] * parts[1][2]) / (w[0] * parts[0][1] + w[1] * parts[1][1])[:, None]
    assert np.max(np.abs(whole - merged)) <= 1e-12 * np.max(np.abs(whole))
    assert np.array_equal(_dec(tb, enc, q, 4, 172, empty, empty), model.decode_buffered(
        tb, 0, 0, q, enc["k_tiles"], enc["k_norms"], enc["v_tiles"], enc["v_norm"], 4, 172, empty, empty))
