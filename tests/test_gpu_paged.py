"""Paged cache (PagedAttention's block table, cited on the blockgtq pages):
the same kernels through a page-id indirection.  A paged state and a
contiguous one fed the same rows must hold the same tile bytes (page for
tile) and give bit-identical decode results; the paged decode matches the
oracle on an uploaded cache; bad page ids raise the device flag."""
import numpy as np
import pytest
import torch

from oracle import model
from packed_decode_attention_b200 import bgtq
from packed_decode_attention_b200 import workloads as wl
from parity_helpers import REL_TOL, library_config, oracle_config, row_rel_err

pytestmark = pytest.mark.gpu

DEVERR_PAGE = 32


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return torch.device("cuda:0")


def _block_table(lens, n_tiles_cap, extra, rng):
    """Shuffled page ids for every tile each sequence may reach (len + extra);
    other entries -1.  Returns (table int32 [B, T], pool size)."""
    need = [(n + extra + 63) // 64 for n in lens]
    pool = sum(need) + 3                     # a few pages nobody owns
    ids = rng.permutation(pool)
    table = np.full((len(lens), n_tiles_cap), -1, dtype=np.int32)
    k = 0
    for b, nt in enumerate(need):
        table[b, :nt] = ids[k:k + nt]
        k += nt
    return table, pool


def _fill(kv, w, lens, dev, chunk):
    """Prefill through the library in chunks that start inside tiles."""
    B = len(lens)
    for layer in range(w.n_layers):
        for b, ln in enumerate(lens):
            for s0 in range(0, ln, chunk):
                n = min(chunk, ln - s0)
                kk = torch.zeros((1, B, n, w.n_kv_heads, 128), dtype=torch.float16, device=dev)
                vv = torch.zeros_like(kk)
                kk[0, b] = wl.keys(w, layer, b, s0, n, device=dev)
                vv[0, b] = wl.values(w, layer, b, s0, n, device=dev)
                start = torch.zeros(B, dtype=torch.int32, device=dev)
                count = torch.zeros(B, dtype=torch.int32, device=dev)
                start[b] = s0
                count[b] = n
                kv.encode_append(layer, kk, vv, start, count)


def _append_one(kv, w, lens, dev):
    """One decode-time row per sequence at position len (the few-row path)."""
    B = len(lens)
    for layer in range(w.n_layers):
        kk = torch.stack([wl.keys(w, layer, b, lens[b], 1, device=dev) for b in range(B)])[None]
        vv = torch.stack([wl.values(w, layer, b, lens[b], 1, device=dev) for b in range(B)])[None]
        kv.encode_append(layer, kk, vv, torch.tensor(lens, dtype=torch.int32, device=dev),
                         torch.ones(B, dtype=torch.int32, device=dev))


@pytest.mark.parametrize("kbits,vbits", [(3, 3), (3, 2), (2, 2)])
def test_paged_equals_contiguous(dev, kbits, vbits):
    lens = [700, 1300, 64, 129]
    extra = 3
    w = wl.scaled(wl.WORKLOADS["tiny"], n_layers=2, n_kv_heads=2, n_q_heads=8, batch=len(lens),
                  seq_len=max(lens) + extra, k_bits=kbits, v_bits=vbits, n_calib=64)
    rng = np.random.default_rng(kbits * 10 + vbits)
    T = (w.seq_len + 63) // 64
    table, pool = _block_table(lens, T, extra, rng)
    cq, ck = wl.calibration(w, device=dev)
    cont = bgtq.PackedKVCache(library_config(w), dev)
    paged = bgtq.PackedKVCache(library_config(w, page_pool_tiles=pool), dev)
    assert paged.cache_bytes < cont.cache_bytes
    bt = torch.from_numpy(table).to(dev)
    paged.set_block_table(bt)
    for kv in (cont, paged):
        kv.allocate(cq, ck)
        _fill(kv, w, lens, dev, chunk=500)
    cur = list(lens)
    for _ in range(extra):
        for kv in (cont, paged):
            _append_one(kv, w, cur, dev)
        cur = [n + 1 for n in cur]
    torch.cuda.synchronize()
    assert cont.device_error() == 0 and paged.device_error() == 0
    # tile bytes and norms, page for tile
    for layer in range(w.n_layers):
        for b, n in enumerate(cur):
            nt = (n + 63) // 64
            for h in range(w.n_kv_heads):
                pages = bt[b, :nt].long()
                assert torch.equal(cont.k_tiles()[layer, b, h, :nt], paged.k_tiles()[layer, h][pages])
                assert torch.equal(cont.v_tiles()[layer, b, h, :nt], paged.v_tiles()[layer, h][pages])
                kn_p = paged.k_norms()[layer, h].view(pool, 64, 4)[pages].reshape(-1, 4)[:n]
                vn_p = paged.v_norms()[layer, h].view(pool, 64)[pages].reshape(-1)[:n]
                assert torch.equal(cont.k_norms()[layer, b, h, :n], kn_p)
                assert torch.equal(cont.v_norms()[layer, b, h, :n], vn_p)
    # decode, all layers per call and one layer per call
    seq = torch.tensor(cur, dtype=torch.int32, device=dev)
    q = torch.stack([wl.decode_query(w, l, cur, device=dev) for l in range(w.n_layers)])
    for path in (0, 1):  # three launches, then the fused launch
        outs = []
        for kv in (cont, paged):
            kv.set_decode_path(path)
            o = torch.empty_like(q)
            kv.decode_attn(0, q, seq, o, layer_count=w.n_layers)
            o1 = torch.empty_like(q)
            for l in range(w.n_layers):
                kv.decode_attn(l, q[l:l + 1], seq, o1[l:l + 1])
            outs.append((o, o1))
        torch.cuda.synchronize()
        assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1]), path
        assert torch.isfinite(outs[0][0].float()).all()
    # buffered decode: 4 sink rows and the last 32 positions as fp16 rows
    lo = torch.full((len(cur),), 4, dtype=torch.int32, device=dev)
    hi = torch.tensor([max(4, n - 32) for n in cur], dtype=torch.int32, device=dev)
    bk = torch.randn((w.n_layers, len(cur), 36, w.n_kv_heads, 128), device=dev).half()
    bv = torch.randn_like(bk)
    cnt = torch.full((len(cur),), 36, dtype=torch.int32, device=dev)
    bufs = []
    for kv in (cont, paged):
        o = torch.empty_like(q)
        kv.decode_attn_buffered(0, q, hi, lo, bk, bv, cnt, o, layer_count=w.n_layers)
        bufs.append(o)
    # logit MAE over a window that crosses pages
    m = 300
    qd = torch.stack([wl.queries(w, l, 1, torch.arange(900, 900 + m), tag=3, device=dev) for l in range(w.n_layers)])
    kd = torch.stack([wl.keys(w, l, 1, 900, m, device=dev) for l in range(w.n_layers)])
    maes = []
    for kv in (cont, paged):
        o = torch.zeros((w.n_layers, w.n_q_heads), dtype=torch.float64, device=dev)
        kv.logit_mae(0, 1, 900, qd, kd, o, layer_count=w.n_layers)
        maes.append(o)
    torch.cuda.synchronize()
    assert torch.equal(bufs[0], bufs[1])
    torch.testing.assert_close(maes[0], maes[1], rtol=1e-9, atol=0)
    assert cont.device_error() == 0 and paged.device_error() == 0
    cont.close()
    paged.close()


def test_paged_decode_matches_oracle(dev):
    """Oracle-encoded rows uploaded into shuffled pages; decode against the oracle."""
    lens = [300, 1000, 65]
    w = wl.scaled(wl.WORKLOADS["tiny"], n_kv_heads=2, n_q_heads=16, batch=len(lens), seq_len=1024, n_calib=64)
    rng = np.random.default_rng(4)
    table, pool = _block_table(lens, 16, 0, rng)
    cfg = library_config(w, page_pool_tiles=pool)
    kv = bgtq.PackedKVCache(cfg, dev)
    ocfg = oracle_config(cfg)
    cq, ck = wl.calibration(w)
    widths = model.allocate(ocfg, cq.numpy(), ck.numpy())
    kv.set_allocation(widths.astype(np.int8))
    kv.set_block_table(torch.from_numpy(table).to(dev))
    tb = model.Tables(ocfg, widths)
    encs = {}
    for b, n in enumerate(lens):
        k = wl.keys(w, 0, b, 0, n)
        v = wl.values(w, 0, b, 0, n)
        nt = (n + 63) // 64
        pages = torch.from_numpy(table[b, :nt].astype(np.int64))
        for h in range(w.n_kv_heads):
            enc = model.encode_rows(tb, 0, h, k[:, h].numpy(), v[:, h].numpy())
            encs[b, h] = enc
            kn = torch.zeros((nt * 64, 4), dtype=torch.float16)
            vn = torch.zeros(nt * 64, dtype=torch.float16)
            kn[:n] = torch.from_numpy(enc["k_norms"])
            vn[:n] = torch.from_numpy(enc["v_norm"])
            kv.k_tiles()[0, h][pages.to(dev)] = torch.from_numpy(enc["k_tiles"]).to(dev)
            kv.v_tiles()[0, h][pages.to(dev)] = torch.from_numpy(enc["v_tiles"]).to(dev)
            kv.k_norms()[0, h].view(pool, 64, 4)[pages.to(dev)] = kn.view(nt, 64, 4).to(dev)
            kv.v_norms()[0, h].view(pool, 64)[pages.to(dev)] = vn.view(nt, 64).to(dev)
    q = wl.decode_query(w, 0, lens)
    g = w.group
    for path in (0, 1):  # three launches, then the fused launch
        kv.set_decode_path(path)
        out = torch.empty((1, len(lens), w.n_q_heads, 128), dtype=torch.float16, device=dev)
        kv.decode_attn(0, q[None].to(dev), torch.tensor(lens, dtype=torch.int32, device=dev), out)
        torch.cuda.synchronize()
        assert kv.device_error() == 0
        got = out[0].float().cpu().numpy()
        for (b, h), enc in encs.items():
            ref = model.decode(tb, 0, h, q[b, h * g:(h + 1) * g].numpy(), enc["k_tiles"], enc["k_norms"],
                               enc["v_tiles"], enc["v_norm"], lens[b])
            assert np.all(row_rel_err(got[b, h * g:(h + 1) * g], ref) <= REL_TOL), (path, b, h)
    kv.close()


def test_bad_page_ids_raise_the_flag(dev):
    """Page ids outside the pool, made on the host: encode skips the tile,
    decode reads page 0 instead; both raise BGTQ_DEVERR_PAGE."""
    w = wl.scaled(wl.WORKLOADS["tiny"], batch=2, seq_len=256, n_calib=64)
    pool = 6
    kv = bgtq.PackedKVCache(library_config(w, page_pool_tiles=pool), dev)
    kv.set_allocation(np.full((1, 1, 64), 3, dtype=np.int8))
    table = torch.tensor([[0, 1, 2, pool + 7], [3, -2, 4, 5]], dtype=torch.int32, device=dev)
    kv.set_block_table(table)
    before = kv.cache.clone()
    kk = torch.ones((1, 2, 64, 1, 128), dtype=torch.float16, device=dev)
    # sequence 0 writes tile 3 (bad id), sequence 1 writes tile 1 (bad id)
    kv.encode_append(0, kk, kk, torch.tensor([192, 64], dtype=torch.int32, device=dev),
                     torch.tensor([64, 64], dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    assert kv.device_error() & DEVERR_PAGE
    assert torch.equal(kv.cache, before)
    q = torch.ones((1, 2, 4, 128), dtype=torch.float16, device=dev)
    out = torch.empty_like(q)
    kv.decode_attn(0, q, torch.tensor([256, 128], dtype=torch.int32, device=dev), out)
    torch.cuda.synchronize()
    assert kv.device_error() & DEVERR_PAGE
    assert torch.isfinite(out.float()).all()
    kv.close()


def test_paged_needs_a_block_table(dev):
    w = wl.scaled(wl.WORKLOADS["tiny"], seq_len=256, n_calib=64)
    kv = bgtq.PackedKVCache(library_config(w, page_pool_tiles=4), dev)
    kv.set_allocation(np.full((1, 1, 64), 3, dtype=np.int8))
    q = torch.ones((1, 1, 4, 128), dtype=torch.float16, device=dev)
    with pytest.raises(bgtq.BgtqError):
        kv.decode_attn(0, q, torch.tensor([64], dtype=torch.int32, device=dev), torch.empty_like(q))
    kv.close()
    cont = bgtq.PackedKVCache(library_config(w), dev)
    with pytest.raises(bgtq.BgtqError):
        cont.set_block_table(torch.zeros((1, 4), dtype=torch.int32, device=dev))
    cont.close()
