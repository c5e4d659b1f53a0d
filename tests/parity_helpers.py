"""Shared helpers for the GPU parity tests: run the library and the oracle on
the same seeded inputs and compare.  The oracle builds its own allocation and
tables from the same calibration rows; no oracle input comes from the GPU."""
import numpy as np
import torch

from oracle import lloyd_max, model, tiles, tqmse
from packed_decode_attention_b200 import bgtq
from packed_decode_attention_b200 import workloads as wl

REL_TOL = 2e-3          # max_i |o - r| / max_i |r| per (sequence, query head) row
CODE_AGREEMENT = 0.9999
THRESHOLD_SLACK = 1e-5


def library_config(w, **over):
    d = dict(n_layers=w.n_layers, n_kv_heads=w.n_kv_heads, n_q_heads=w.n_q_heads, max_batch=w.batch,
             capacity_tokens=w.seq_len, k_avg_bits=w.k_bits, v_avg_bits=w.v_bits, seed=w.seed)
    d.update(over)
    return bgtq.Config(**d)


def oracle_config(cfg):
    return model.Config(cfg.n_layers, cfg.n_kv_heads, cfg.n_q_heads, 128, cfg.k_avg_bits, cfg.v_avg_bits,
                        cfg.b_min, cfg.b_max, cfg.rope_pairing, cfg.seed)


def row_rel_err(got, ref):
    """Per-row max |got - ref| / max |ref| over the last axis."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.max(np.abs(got - ref), axis=-1)
    den = np.max(np.abs(ref), axis=-1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


def compare_codes(gpu_codes, ora_codes, ora_u, widths_per_pos):
    """(agreement fraction, all mismatches within THRESHOLD_SLACK of a threshold)."""
    eq = gpu_codes == ora_codes
    frac = eq.mean()
    ok = True
    bad = np.argwhere(~eq)
    for r, p in bad:
        b = int(widths_per_pos[p])
        th = lloyd_max.codebook_fp16(b)[1].astype(np.float64)
        if np.min(np.abs(th - ora_u[r, p])) > THRESHOLD_SLACK or abs(int(gpu_codes[r, p]) - int(ora_codes[r, p])) != 1:
            ok = False
    return frac, ok, len(bad)


def oracle_u(tables, layer, head, rows, kind):
    """The oracle's unrounded u values [n, positions] in record order."""
    x = np.asarray(rows, dtype=np.float16).astype(np.float64)
    if kind == 0:
        parts = [tqmse.rotated_normalised(x, dims, tables.k_rot[layer, head][b])[0]
                 for b, dims in tables.groups[layer, head]]
        return np.concatenate(parts, axis=1)
    return tqmse.rotated_normalised(x, np.arange(128), tables.v_rot[layer, head])[0]


def fp16_ulp_apart(a, b):
    """Elementwise |a - b| in fp16 ulps (same-sign finite values)."""
    ai = np.asarray(a, dtype=np.float16).view(np.int16).astype(np.int64)
    bi = np.asarray(b, dtype=np.float16).view(np.int16).astype(np.int64)
    return np.abs(ai - bi)


def upload_oracle_rows(kv, layer, seq, head, enc):
    """Write the oracle's packed tiles and norms (positions 0..n-1) into the library's cache."""
    n = enc["n"]
    nt = enc["k_tiles"].shape[0]
    kv.k_tiles()[layer, seq, head, :nt].copy_(torch.from_numpy(enc["k_tiles"]))
    kv.v_tiles()[layer, seq, head, :nt].copy_(torch.from_numpy(enc["v_tiles"]))
    kv.k_norms()[layer, seq, head, :n].copy_(torch.from_numpy(enc["k_norms"]))
    kv.v_norms()[layer, seq, head, :n].copy_(torch.from_numpy(enc["v_norm"]))


def gpu_codes(kv, tb, layer, seq, head, n, vbits):
    """The library's K and V codes of positions 0..n-1, unpacked with the oracle's tile definition."""
    nt = (n + 63) // 64
    kt = kv.k_tiles()[layer, seq, head, :nt].cpu().numpy()
    vt = kv.v_tiles()[layer, seq, head, :nt].cpu().numpy()
    return (tiles.unpack_k_tiles(kt, tb.groups[layer, head], n), tiles.unpack_v_tiles(vt, vbits, n), kt, vt)


def encode_on_gpu(kv, w, layers, lens, dev, chunk=1 << 16):
    """Encode every sequence's keys/values [0, len) of the given layers through the library."""
    for layer in layers:
        for b, ln in enumerate(lens):
            for s0 in range(0, ln, chunk):
                n = min(chunk, ln - s0)
                k = wl.keys(w, layer, b, s0, n, device=dev)
                v = wl.values(w, layer, b, s0, n, device=dev)
                kk = torch.zeros((1, w.batch, n, w.n_kv_heads, 128), dtype=torch.float16, device=dev)
                vv = torch.zeros_like(kk)
                kk[0, b] = k
                vv[0, b] = v
                start = torch.zeros(w.batch, dtype=torch.int32, device=dev)
                count = torch.zeros(w.batch, dtype=torch.int32, device=dev)
                start[b] = s0
                count[b] = n
                kv.encode_append(layer, kk, vv, start, count)
