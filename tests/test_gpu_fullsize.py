"""Parity at the benchmark's full sizes and launch configuration.

llama (1 layer x 8 KV heads, 32768 tokens, K2V2), qwen3b (36 layers x 2 KV
heads, 131072 tokens), batch (28 layers x 4 KV
heads, 16 ragged sequences of 16K-32K) and long (36 layers x 2 KV heads,
524288 tokens): the cache is built and decoded exactly as bench.py does
(same config, chunked prefill, per-layer and all-layers decode calls with the
automatic split).  Checked:
  * every layer's allocation bit-exact against the oracle (energies exact on
    sampled layers);
  * codes of sampled (layer, sequence, head) triples against the oracle's
    encode (>= 99.99 % equal, mismatches one code apart within 1e-5 of a
    threshold);
  * decode: the sampled triples' caches are replaced by the oracle's packed
    tiles (identical caches) and every layer is decoded; sampled heads must
    match the oracle within 2e-3, all others must be finite and agree
    between the per-layer and the all-layers launch.
"""
import numpy as np
import pytest
import torch

from oracle import energy as oenergy
from oracle import model, tqmse
from packed_decode_attention_b200 import bgtq
from packed_decode_attention_b200 import workloads as wl

from parity_helpers import (CODE_AGREEMENT, REL_TOL, compare_codes, fp16_ulp_apart, gpu_codes, oracle_u,
                            row_rel_err, upload_oracle_rows)

pytestmark = pytest.mark.gpu

SAMPLES = {
    # (layer, sequence) pairs checked against the oracle; all KV heads of each
    "llama": [(0, 0)],
    "qwen3b": [(0, 0), (17, 0), (35, 0)],
    # the ragged batch: its first and last sequences, the shortest (1), the
    # longest (10) and two of middle length (4, 7)
    "batch": [(0, 0), (20, 1), (9, 4), (13, 7), (5, 10), (27, 15)],
    "long": [(35, 0)],
}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    bgtq.lib()
    return torch.device("cuda:0")


@pytest.mark.parametrize("name", ["llama", "qwen3b", "batch", "long"])
def test_full_size_parity(dev, name):
    w = wl.WORKLOADS[name]
    lens = wl.seq_lens(w)
    cfg = bgtq.Config(**wl.bench_config_fields(w))
    kv = bgtq.PackedKVCache(cfg, dev)
    cq, ck = wl.calibration(w, device=dev)
    kv.allocate(cq, ck)
    ocfg = model.Config(cfg.n_layers, cfg.n_kv_heads, cfg.n_q_heads, 128, cfg.k_avg_bits, cfg.v_avg_bits,
                        cfg.b_min, cfg.b_max, cfg.rope_pairing, cfg.seed)
    cq, ck = cq.cpu().numpy(), ck.cpu().numpy()
    widths = model.allocate(ocfg, cq, ck)
    assert np.array_equal(kv.get_allocation().astype(np.int64), widths)
    eq, ek = bgtq.bgtq_get_energy(kv.state, cfg.n_layers, cfg.n_kv_heads)
    for l in sorted({l for l, _ in SAMPLES[name]}):
        oq, ok = oenergy.block_energies(cq[l], ck[l], 0)
        assert eq[l] == oq and ek[l] == ok
    del cq, ck

    sampled = set(SAMPLES[name])
    rows = {}

    def keep(layer, b, s0, k, v):
        if (layer, b) in sampled:
            rows.setdefault((layer, b), []).append((s0, k.cpu().numpy(), v.cpu().numpy()))

    wl.prefill(kv, w, lens, dev, on_chunk=keep)
    torch.cuda.synchronize()
    assert kv.device_error() == 0

    tb = model.Tables(ocfg, widths, layers=sorted({l for l, _ in sampled}))
    q_all = torch.stack([wl.decode_query(w, l, lens, device=dev) for l in range(w.n_layers)])
    encs = {}
    for (l, b), parts in rows.items():
        parts.sort(key=lambda x: x[0])
        k = np.concatenate([p[1] for p in parts])
        v = np.concatenate([p[2] for p in parts])
        n = lens[b]
        assert k.shape[0] == n
        for h in range(w.n_kv_heads):
            enc = model.encode_rows(tb, l, h, k[:, h], v[:, h])
            g_kc, g_vc, _, _ = gpu_codes(kv, tb, l, b, h, n, cfg.v_avg_bits)
            wpos = tqmse.record_widths(tb.groups[l, h])
            # u only where codes differ (the full u arrays are large)
            for gc, oc, kind, x, wp in ((g_kc, enc["k_codes"], 0, k[:, h], wpos),
                                        (g_vc, enc["v_codes"], 1, v[:, h], np.full(128, cfg.v_avg_bits))):
                bad_rows = np.nonzero(np.any(gc != oc, axis=1))[0]
                frac = 1.0 - np.count_nonzero(gc != oc) / gc.size
                assert frac >= CODE_AGREEMENT, (name, l, b, h, kind, frac)
                if len(bad_rows):
                    u = oracle_u(tb, l, h, x[bad_rows], kind)
                    _, ok_, _ = compare_codes(gc[bad_rows], oc[bad_rows], u, wp)
                    assert ok_, (name, l, b, h, kind)
            assert np.all(fp16_ulp_apart(kv.k_norms()[l, b, h, :n].cpu().numpy(), enc["k_norms"]) <= 1)
            assert np.all(fp16_ulp_apart(kv.v_norms()[l, b, h, :n].cpu().numpy(), enc["v_norm"]) <= 1)
            upload_oracle_rows(kv, l, b, h, enc)
            encs[l, b, h] = enc
    del rows

    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    g = w.group
    qh = q_all.cpu().numpy()
    refs = {(l, b, h): model.decode(tb, l, h, qh[l, b, h * g:(h + 1) * g], enc["k_tiles"], enc["k_norms"],
                                    enc["v_tiles"], enc["v_norm"], enc["n"]) for (l, b, h), enc in encs.items()}
    # both decode paths: three launches (rotation, split pass, combine) and the fused launch
    for path in (0, 1):
        kv.set_decode_path(path)
        out_layer = torch.empty((w.n_layers, w.batch, w.n_q_heads, 128), dtype=torch.float16, device=dev)
        for l in range(w.n_layers):
            kv.decode_attn(l, q_all[l:l + 1], seq, out_layer[l:l + 1])
        out_all = torch.empty_like(out_layer)
        kv.decode_attn(0, q_all, seq, out_all, layer_count=w.n_layers)
        # the benchmark's call (decode_step, here with no new row) is the same computation
        out_step = torch.empty_like(out_layer)
        for l in range(w.n_layers):
            kv.decode_step(l, None, None, None, None, q_all[l:l + 1], seq, out_step[l:l + 1])
        torch.cuda.synchronize()
        assert kv.device_error() == 0
        assert torch.equal(out_step, out_layer), path
        assert torch.isfinite(out_layer.float()).all() and torch.isfinite(out_all.float()).all()
        a = out_layer.float().cpu().numpy()
        assert np.all(row_rel_err(out_all.float().cpu().numpy(), a) <= REL_TOL), path
        for (l, b, h), ref in refs.items():
            err = row_rel_err(a[l, b, h * g:(h + 1) * g], ref)
            assert np.all(err <= REL_TOL), (name, path, l, b, h, err.max())
    kv.close()
